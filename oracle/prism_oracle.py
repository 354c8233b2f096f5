"""Plain fp64 CPU oracle for Prism's block-importance estimator and the
block-sparse causal attention that consumes its mask.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module.  It shares no code with
the CUDA path and must never be used as a fallback for it.

Source: "Prism: Spectral-Aware Block-Sparse Attention" (Wang et al., 2026,
arXiv 2602.08426).  Citations name the web page and the passage:

* [review:method]   paper.rainbus.top review, paragraph listing the full
                    pipeline, steps (1)-(7).
* [review:novelty]  paper.rainbus.top review, novelty paragraph (closed form
                    lambda_j(B) ~ sinc(B theta_j / 2 pi), three spectral zones).
* [review:repro]    paper.rainbus.top review, reproducibility paragraph
                    (B = 128, d_high = 64, d_low = 96, p = 0.95 / 0.93).
* [summary:1]..[summary:4]  gist.science "Technical Summary", sections 1
                    (problem / blind spot), 2A (dual band), 2B (RMS-based
                    temperature calibration), 4 (results).

The method is a heuristic, so the oracle restates its steps in the pages'
order and notation, in fp64 throughout:

  (1) spectral slicing of Q, K into a high band and a low band;
  (2) mean pooling of each band per block of B tokens -> Q_bar_z, K_bar_z;
  (3) RMS of each pooled band (spectral energy density);
  (4) temperature tau_z from those RMS values;
  (5) S_bar_z = softmax(Q_bar_z K_bar_z^T / (tau_z sqrt(d_z))), causal over blocks;
  (6) Top-P per query-block row and band -> M_z;
  (7) M = M_high OR M_low;
  then block-sparse causal attention restricted to M.

Readings taken where the pages are silent (each one is listed in the design
notes with its reason):

* tau_z (step 4) is not printed.  Reading R1: tau_z = (RMS(Q_bar_z) *
  RMS(K_bar_z)) / (RMS(Q_bar_full) * RMS(K_bar_full)); dividing the band
  logits by tau_z rescales their magnitude to that of the full-spectrum pooled
  logits ([review:method] step 4, [summary:2B]).  If any RMS is 0, tau = 1.
  Parity of the absolute tau values against the paper: unpinned (no worked
  example is printed).
* RMS granularity: one scalar per (batch, head, band) over all blocks.
* Causal scope at block level: softmax over key blocks j <= i; the diagonal
  block uses its full pooled K_bar.
* Top-P: rank key blocks by (-prob, j) (ties -> lower block index first);
  keep a block iff the mass strictly ahead of it is < p (nucleus rule, the
  crossing block is kept); p >= 1 keeps every causal block.
* GQA: Q head h reads KV head h // (Hq / Hkv).
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence

import numpy as np


# --------------------------------------------------------------------------
# steps (1)-(2): slicing and mean pooling        [review:method] steps 1-2
# --------------------------------------------------------------------------
def to_f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> fp64 numpy (exact upcast)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: the oracle itself needs only numpy
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def band_slice(x: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """Step (1): the columns of the last axis that belong to a band."""
    return x[..., list(dims)]


def mean_pool(x: np.ndarray, block: int) -> np.ndarray:
    """Step (2): mean over each run of ``block`` tokens on axis -2.

    x [..., N, d] -> [..., ceil(N / block), d].  When N is not a multiple of
    block, the last block is the mean over the tokens it has (the pages define
    blocks of B tokens only; this is the plainest reading for a short tail).
    """
    n = x.shape[-2]
    nb = -(-n // block)
    full = (n // block) * block
    shp = x.shape[:-2] + (n // block, block, x.shape[-1])
    head = x[..., :full, :].reshape(shp).mean(axis=-2)
    if full == n:
        return head
    tail = x[..., full:, :].mean(axis=-2, keepdims=True)
    out = np.concatenate([head, tail], axis=-2)
    assert out.shape[-2] == nb
    return out


# --------------------------------------------------------------------------
# step (3): RMS of the pooled bands               [review:method] step 3
# --------------------------------------------------------------------------
def rms(pooled_band: np.ndarray) -> np.ndarray:
    """Root mean square over the (block, dim) entries of one head's pooled band.

    pooled_band [..., nb, d_z] -> [...].
    """
    return np.sqrt(np.mean(pooled_band * pooled_band, axis=(-2, -1)))


# --------------------------------------------------------------------------
# step (4): temperatures                          [review:method] step 4, [summary:2B]
# --------------------------------------------------------------------------
def tau_rms(rq_z: float, rk_z: float, rq_full: float, rk_full: float) -> float:
    """Reading R1 of the temperature: the ratio of the band's pooled energy
    (Q RMS times K RMS) to the full spectrum's; 1 when any factor is 0."""
    num = rq_z * rk_z
    den = rq_full * rk_full
    if num == 0.0 or den == 0.0:
        return 1.0
    return num / den


# --------------------------------------------------------------------------
# step (5): dual-band scoring                     [review:method] step 5
# --------------------------------------------------------------------------
def band_logits(qbar_z: np.ndarray, kbar_z: np.ndarray, tau_z: float) -> np.ndarray:
    """Q_bar_z K_bar_z^T / (tau_z sqrt(d_z)) with key blocks j > i set to -inf.

    qbar_z [nb, d_z], kbar_z [nb, d_z] -> [nb, nb].
    """
    d_z = qbar_z.shape[-1]
    lg = (qbar_z @ kbar_z.T) / (tau_z * math.sqrt(d_z))
    nb = lg.shape[0]
    lg[np.triu_indices(nb, k=1)] = -np.inf
    return lg


def softmax_rows(logits: np.ndarray) -> np.ndarray:
    """Row softmax (max-subtracted); -inf entries get probability 0."""
    m = np.max(logits, axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / np.sum(e, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# step (6): Top-P                                 [review:method] step 6
# --------------------------------------------------------------------------
def top_p(probs: np.ndarray, p: float):
    """Top-P per row over the causal entries j <= i.

    probs [nb, nb] (rows sum to 1 over j <= i).  Returns (keep [nb, nb] bool,
    c_excl [nb, nb]) where c_excl[i, j] is the probability mass ranked strictly
    ahead of block j in row i under the order (-prob, j); it is the quantity the
    keep decision compares with p.  Entries above the diagonal: keep False,
    c_excl +inf.
    """
    nb = probs.shape[0]
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    key = np.where(causal, -probs, np.inf)
    order = np.argsort(key, axis=1, kind="stable")  # stable: ties -> lower j first
    sorted_p = np.take_along_axis(np.where(causal, probs, 0.0), order, axis=1)
    c_incl = np.cumsum(sorted_p, axis=1)
    c_excl_sorted = np.concatenate([np.zeros((nb, 1)), c_incl[:, :-1]], axis=1)
    c_excl = np.empty_like(c_excl_sorted)
    np.put_along_axis(c_excl, order, c_excl_sorted, axis=1)
    c_excl = np.where(causal, c_excl, np.inf)
    if p >= 1.0:
        keep = causal.copy()
    else:
        keep = causal & (c_excl < p)
    return keep, c_excl


# --------------------------------------------------------------------------
# the whole estimator, steps (1)-(7)
# --------------------------------------------------------------------------
def estimate_head(qbar_hi, qbar_lo, qbar_full, kbar_hi, kbar_lo, kbar_full, p,
                  tau_mode="rms", tau_explicit=(1.0, 1.0)) -> Dict[str, np.ndarray]:
    """Steps (3)-(7) for one (batch, Q head) given its pooled bands and the pooled
    bands of its KV head."""
    if tau_mode == "rms":
        rq = dict(hi=rms(qbar_hi), lo=rms(qbar_lo), full=rms(qbar_full))
        rk = dict(hi=rms(kbar_hi), lo=rms(kbar_lo), full=rms(kbar_full))
        tau_hi = tau_rms(rq["hi"], rk["hi"], rq["full"], rk["full"])
        tau_lo = tau_rms(rq["lo"], rk["lo"], rq["full"], rk["full"])
    else:
        tau_hi, tau_lo = float(tau_explicit[0]), float(tau_explicit[1])
    lg_hi = band_logits(qbar_hi, kbar_hi, tau_hi)
    lg_lo = band_logits(qbar_lo, kbar_lo, tau_lo)
    pr_hi = softmax_rows(lg_hi)
    pr_lo = softmax_rows(lg_lo)
    keep_hi, cx_hi = top_p(pr_hi, p)
    keep_lo, cx_lo = top_p(pr_lo, p)
    return dict(tau=np.array([tau_hi, tau_lo]),
                logits=np.stack([lg_hi, lg_lo]), probs=np.stack([pr_hi, pr_lo]),
                c_excl=np.stack([cx_hi, cx_lo]), keep_hi=keep_hi, keep_lo=keep_lo,
                mask=keep_hi | keep_lo)  # step (7): union


def estimate(q, k, band_hi: Sequence[int], band_lo: Sequence[int], p: float,
             block: int = 128, tau_mode: str = "rms", tau_explicit=(1.0, 1.0),
             heads: Optional[Iterable[int]] = None, keep_dense: bool = True,
             force_sink: bool = False, force_diag: bool = False):
    """Prism's estimator on q [b, Hq, N, D], k [b, Hkv, N, D] (post-RoPE).

    force_sink / force_diag: optional additions to the mask after step (7),
    key block 0 / the diagonal block of every row (off by default: the method's
    mask is exactly M_high | M_low).

    Returns a dict of fp64/bool arrays with a leading [b, Hq'] (Hq' = the
    selected heads):  q_pool [.., nb, D], tau [.., 2], logits / probs / c_excl
    [.., 2, nb, nb], keep_hi / keep_lo / mask [.., nb, nb]; plus k_pool
    [b, Hkv, nb, D] and the RMS values rms_q [b, Hq', 3], rms_k [b, Hkv, 3]
    (hi, lo, full).
    """
    qf = to_f64(q)
    kf = to_f64(k)
    b, hq, n, d = qf.shape
    hkv = kf.shape[1]
    assert hq % hkv == 0
    grp = hq // hkv
    heads = list(range(hq)) if heads is None else list(heads)
    full = list(range(d))
    out: Dict[str, list] = {key: [] for key in
                            ("q_pool", "tau", "logits", "probs", "c_excl",
                             "keep_hi", "keep_lo", "mask", "rms_q")}
    k_pool_all, rms_k_all = [], []
    for bi in range(b):
        # steps (1)-(2) for the keys, once per KV head
        kb = {}
        for kv in range(hkv):
            kb[kv] = (mean_pool(band_slice(kf[bi, kv], band_hi), block),
                      mean_pool(band_slice(kf[bi, kv], band_lo), block),
                      mean_pool(band_slice(kf[bi, kv], full), block))
        k_pool_all.append(np.stack([kb[kv][2] for kv in range(hkv)]))
        rms_k_all.append(np.array([[rms(kb[kv][0]), rms(kb[kv][1]), rms(kb[kv][2])]
                                   for kv in range(hkv)]))
        rows = {key: [] for key in out}
        for h in heads:
            qh = qf[bi, h]
            qb_hi = mean_pool(band_slice(qh, band_hi), block)
            qb_lo = mean_pool(band_slice(qh, band_lo), block)
            qb_full = mean_pool(band_slice(qh, full), block)
            kv = h // grp
            res = estimate_head(qb_hi, qb_lo, qb_full, *kb[kv], p, tau_mode, tau_explicit)
            if force_sink or force_diag:
                # optional additions after the union (not part of the method)
                nbh = res["mask"].shape[0]
                forced = np.zeros((nbh, nbh), dtype=bool)
                if force_sink:
                    forced[:, 0] = True
                if force_diag:
                    forced[np.arange(nbh), np.arange(nbh)] = True
                res["mask"] = res["mask"] | forced
            rows["q_pool"].append(qb_full)
            rows["rms_q"].append(np.array([rms(qb_hi), rms(qb_lo), rms(qb_full)]))
            for key in ("tau", "logits", "probs", "c_excl", "keep_hi", "keep_lo", "mask"):
                if not keep_dense and key in ("logits", "probs"):
                    continue
                rows[key].append(res[key])
        for key in out:
            if rows[key]:
                out[key].append(np.stack(rows[key]))
    res = {key: np.stack(val) for key, val in out.items() if val}
    res["k_pool"] = np.stack(k_pool_all)
    res["rms_k"] = np.stack(rms_k_all)
    return res


# --------------------------------------------------------------------------
# block-sparse causal attention          [summary:1] "only computes a subset of
# attention blocks"; token-causal inside the diagonal block
# --------------------------------------------------------------------------
def sparse_attention_block(q, k, v, mask_row: np.ndarray, b: int, h: int, i: int,
                           group: int, block: int = 128,
                           scale: Optional[float] = None) -> np.ndarray:
    """Exact fp64 attention output for the ``block`` queries of query block i of
    (batch b, Q head h), attending only to the key blocks j <= i whose bit is set
    in ``mask_row`` [nb] (bool), with key s <= query t inside block i.

    Returns [rows, D], rows = the tokens block i has (block, or fewer for a
    short last block).  A row with no visible key returns 0.
    """
    n = q.shape[2]
    qf = to_f64(q[b, h, i * block:min((i + 1) * block, n)])
    kv = h // group
    d = qf.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    js = [j for j in range(i + 1) if bool(mask_row[j])]
    if not js:
        return np.zeros((qf.shape[0], d))
    kf = np.concatenate([to_f64(k[b, kv, j * block:min((j + 1) * block, n)]) for j in js])
    vf = np.concatenate([to_f64(v[b, kv, j * block:min((j + 1) * block, n)]) for j in js])
    key_pos = np.concatenate([np.arange(j * block, min((j + 1) * block, n)) for j in js])
    q_pos = np.arange(i * block, i * block + qf.shape[0])
    s = (qf @ kf.T) * scale
    visible = key_pos[None, :] <= q_pos[:, None]
    s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(visible, np.exp(s - m), 0.0)
    den = e.sum(axis=1, keepdims=True)
    out = (e @ vf) / np.where(den > 0, den, 1.0)
    return np.where(den > 0, out, 0.0)


def dense_causal_attention(q, k, v, group: int, scale: Optional[float] = None) -> np.ndarray:
    """Textbook causal attention softmax(Q K^T * scale + causal) V in fp64 for
    small inputs: q [b, Hq, N, D] -> [b, Hq, N, D]."""
    qf, kf, vf = to_f64(q), to_f64(k), to_f64(v)
    b, hq, n, d = qf.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = np.zeros_like(qf)
    causal = np.tril(np.ones((n, n), dtype=bool))
    for bi in range(b):
        for h in range(hq):
            s = qf[bi, h] @ kf[bi, h // group].T * scale
            s = np.where(causal, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            e = np.exp(s)
            out[bi, h] = (e / e.sum(axis=1, keepdims=True)) @ vf[bi, h // group]
    return out


# --------------------------------------------------------------------------
# bit-packed mask format: uint32 words, bit (j % 32) of word j // 32 of row i
# --------------------------------------------------------------------------
def pack_mask(mask: np.ndarray) -> np.ndarray:
    """bool [..., nb, nb] -> uint32 [..., nb, ceil(nb / 32)] (LSB = lower block)."""
    nb = mask.shape[-1]
    words = (nb + 31) // 32
    padded = np.zeros(mask.shape[:-1] + (words * 32,), dtype=np.uint64)
    padded[..., :nb] = mask
    bits = padded.reshape(mask.shape[:-1] + (words, 32))
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (bits * weights).sum(axis=-1).astype(np.uint32)


def unpack_mask(words: np.ndarray, nb: int) -> np.ndarray:
    """uint32 [..., nb, W] -> bool [..., nb, nb]."""
    w = np.asarray(words, dtype=np.uint64)
    shifts = np.arange(32, dtype=np.uint64)
    bits = ((w[..., None] >> shifts) & np.uint64(1)).astype(bool)
    return bits.reshape(w.shape[:-1] + (w.shape[-1] * 32,))[..., :nb]
