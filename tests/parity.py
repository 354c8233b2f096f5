"""Parity rules between the CUDA path and the fp64 oracle (test code only).

Rules (tolerances from the arithmetic of each step):
* pooled block means: |m_gpu - m_ref| <= 2^-18 * (mean of |x| over the
  block's tokens, per dim) (fp32 sums of <= 128 bf16 values in 8
  tensor-core steps: at most ~2^-20 * sum |x| / tokens; 4x margin);
* temperatures: relative 1e-4 (fp32 sums of <= 2^15 non-negative partials);
* band scores L_z: |L_gpu - L_ref| <= 1e-3 * max(|L_ref|, 1e-3 * max_row |L_ref|)
  on the causal entries (fp32 dot products of 64..96 pooled dims);
* masks: bit-exact, except blocks whose oracle decision quantity (the mass
  ranked strictly ahead, c_excl) lies within 1e-4 of p -- those are exempt and
  counted;
* Top-P on the GPU's own weights: bit-exact.  ``topp_fixed_point`` restates
  the GPU's decision rule (ranked by (-e_j, j); block j kept iff the sum of
  round(e_k 2^31) over the blocks ahead of it is < max(floor(p Z), 1)) on the
  e_j the GPU reports, and the GPU mask must equal it bit for bit;
* the oracle's fp64 softmax + Top-P on the GPU's own scores agrees with the
  GPU mask except where its c_excl is within ``SELF_WINDOW`` of p: the GPU's
  e_j carry fp32 errors (the argument L log2 e - max log2 e rounded twice,
  <= 2^-23 |L log2 e| + 2^-24 |max log2 e|, and the hardware exp2's <= 2^-22
  relative error) and 2^-31 fixed-point rounding per block; for |L| <= 50 that
  is <= 2e-6 relative per weight, so c_excl moves by < 1e-5;
* attention output vs the oracle with the same mask: max-abs <= 2e-2 and
  mean-abs <= 2e-3 (bf16 inputs, bf16 P, bf16 output rounding).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_attention_band_b200 as pb
import oracle
from tests import gen

MASK_WINDOW = 1e-4
SELF_WINDOW = 1e-5
POOL_REL = 2.0 ** -18
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3


def make_cfg(w: gen.Workload, bands=None, p=None, **kw) -> pb.PrismConfig:
    hi, lo = bands if bands is not None else gen.default_bands(w.head_dim)
    return pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, w.p if p is None else p, **kw)


def unpack_tri(packed: np.ndarray, nb: int) -> np.ndarray:
    """[..., nb(nb+1)/2] packed lower-triangular rows -> [..., nb, nb] with -inf above."""
    out = np.full(packed.shape[:-1] + (nb, nb), -np.inf)
    il, jl = np.tril_indices(nb)
    out[..., il, jl] = packed  # tril_indices enumerates row by row, j ascending
    return out


def run_estimate(cfg: pb.PrismConfig, q: torch.Tensor, k: torch.Tensor, with_scores=True, extras=None):
    """q, k on the GPU.  Returns (mask bool [b,hq,nb,nb], scores [b,hq,2,nb,nb] or None, tau,
    mask words).  ``extras`` (a dict, optional) receives the GPU's Top-P weights
    ("weights" [b,hq,2,nb,nb], NaN above the diagonal; when p < 1) and pooled
    means ("pooled" [b*hq + b*hkv, nb, 128])."""
    b, hq, hkv = q.shape[0], q.shape[1], k.shape[1]
    nb, W = cfg.nb, cfg.words
    dev = q.device
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
    mask = torch.full((b, hq, nb, W), 0xDEAD, dtype=torch.int32, device=dev)
    tri = nb * (nb + 1) // 2
    scores = torch.empty(b, hq, 2, tri, dtype=torch.float32, device=dev) if with_scores else None
    tau = torch.empty(b, hq, 2, dtype=torch.float32, device=dev)
    weights = pooled = None
    if extras is not None:
        weights = torch.full((b, hq, 2, tri), float("nan"), dtype=torch.float32, device=dev)
        pooled = torch.full((b * (hq + hkv), nb, 128), float("nan"), dtype=torch.float32, device=dev)
    pb.prism_estimate(cfg, q, k, mask, ws, dbg_scores=scores, dbg_tau=tau, dbg_weights=weights,
                      dbg_pooled=pooled)
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    words = mask.cpu().numpy().view(np.uint32)
    m = oracle.unpack_mask(words, nb)
    sc = unpack_tri(scores.cpu().double().numpy(), nb) if with_scores else None
    if extras is not None:
        wt = unpack_tri(weights.cpu().double().numpy(), nb)
        wt[~np.isfinite(wt)] = np.nan  # above the diagonal
        extras["weights"] = wt
        extras["pooled"] = pooled.cpu().double().numpy()
    return m, sc, tau.cpu().double().numpy(), words


def topp_fixed_point(weights: np.ndarray, p: float) -> np.ndarray:
    """The GPU's Top-P decision restated on its own weights.

    weights [..., nb, nb]: the e_j of each causal row (NaN above the
    diagonal; 0 where the exponential underflowed; the maximum 1 up to one
    rounding).  Per row: masses m_j = round-half-even(e_j 2^31) (exact: e_j is
    an fp32 value and the product a power-of-two scaling), Z = sum m_j,
    lim = max(floor(p Z), 1) with p the fp32 value the library uses and the
    product formed in fp64; blocks ranked by (-e_j, j); block j kept iff the
    masses ranked strictly ahead of it sum to < lim.  Returns keep [..., nb, nb]."""
    pf = float(np.float32(p))
    nb = weights.shape[-1]
    flat = weights.reshape(-1, nb, nb)
    out = np.zeros(flat.shape, dtype=bool)
    for r in range(flat.shape[0]):
        for i in range(nb):
            e = flat[r, i, :i + 1]
            # the row maximum's weight is 1 up to the rounding of the shifted
            # argument; the hardware exponential flushes results below 2^-126 to 0
            assert np.all(np.isfinite(e)) and np.all(e >= 0) and np.all(e < 2) and abs(e.max() - 1.0) < 1e-6, \
                "weights must lie in [0, 2) with the row maximum at 1"
            m = np.rint(e * 2.0 ** 31).astype(np.int64)
            z = int(m.sum())
            lim = max(int(np.float64(pf) * np.float64(z)), 1)
            order = np.lexsort((np.arange(i + 1), -e))  # by -e, then j
            ahead = np.concatenate([[0], np.cumsum(m[order])[:-1]])
            keep_sorted = ahead < lim
            out[r, i, order[keep_sorted]] = True
    return out.reshape(weights.shape)


def check_topp_exact(mask_gpu, weights, p, force_sink=False, force_diag=False):
    """The GPU mask equals the union of both bands' fixed-point Top-P on its own weights, bit for bit."""
    keep = topp_fixed_point(weights, p)
    expect = keep[..., 0, :, :] | keep[..., 1, :, :]
    nb = mask_gpu.shape[-1]
    if force_sink:
        expect[..., :, 0] = True
    if force_diag:
        expect[..., np.arange(nb), np.arange(nb)] = True
    diff = expect != mask_gpu
    assert not diff.any(), f"{diff.sum()} mask bits differ from the fixed-point Top-P on the GPU's own weights"


def check_pooled(pooled_gpu: np.ndarray, q, k, seq_tokens=None, only=None):
    """Pooled block means [b*hq + b*hkv, nb, 128] against the oracle's mean_pool
    of the same bf16 inputs, element by element (tolerance in the module
    docstring).  ``seq_tokens``: per-batch token counts (padded layouts); blocks
    past a sequence are not compared.  ``only``: the row indices to check (all
    by default); ``pooled_gpu`` may then hold just those rows, in that order."""
    b, hq, n, _ = q.shape
    hkv = k.shape[1]
    rows = [(q, bi, h) for bi in range(b) for h in range(hq)] + [(k, bi, h) for bi in range(b) for h in range(hkv)]
    sel = list(range(len(rows))) if only is None else list(only)
    compact = only is not None and pooled_gpu.shape[0] == len(sel)
    worst = 0.0
    for pos, r in enumerate(sel):
        x, bi, h = rows[r]
        nt = n if seq_tokens is None else seq_tokens[bi]
        xs = oracle.to_f64(x[bi, h, :nt])
        ref = oracle.mean_pool(xs, 128)
        nbx = ref.shape[0]
        scale = oracle.mean_pool(np.abs(xs), 128)  # mean |x| of each (block, dim)
        got = pooled_gpu[pos if compact else r, :nbx]
        err = np.abs(got - ref)
        bound = POOL_REL * np.maximum(scale, 1e-300)
        bad = err > bound
        assert not bad.any(), (f"pooled row {r}: {bad.sum()} means off (max err {err.max():.3g}, "
                               f"first at block/dim {np.argwhere(bad)[:3].tolist()})")
        worst = max(worst, float((err / bound).max()))
    return worst


def check_tau(tau_gpu, ref, rtol=1e-4):
    np.testing.assert_allclose(tau_gpu, ref["tau"], rtol=rtol)


def check_scores(sc_gpu, ref):
    lr = ref["logits"]
    finite = np.isfinite(lr)
    assert np.array_equal(finite, np.isfinite(sc_gpu)), "causal structure of the scores differs"
    rowmax = np.max(np.where(finite, np.abs(lr), 0.0), axis=-1, keepdims=True)
    tol = 1e-3 * np.maximum(np.abs(lr), 1e-3 * rowmax)
    err = np.abs(np.where(finite, sc_gpu, 0.0) - np.where(finite, lr, 0.0))
    bad = err > np.where(finite, tol, 1.0)
    assert not bad.any(), f"{bad.sum()} score entries outside 1e-3 relative (max err {err.max():.3g})"


def check_mask(mask_gpu, ref, p, window=MASK_WINDOW):
    """Bit-exact except blocks with |c_excl - p| < window in the band that decided.

    Returns (n_mismatch_total, n_exempt)."""
    nb = mask_gpu.shape[-1]
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    assert not np.any(mask_gpu & ~causal), "mask bits above the diagonal"
    diff = mask_gpu != ref["mask"]
    near = np.zeros_like(diff)
    for band in range(2):
        near |= np.abs(ref["c_excl"][..., band, :, :] - p) < window
    unexplained = diff & ~near
    assert not unexplained.any(), (
        f"{unexplained.sum()} mask bits differ outside the {window} window of p "
        f"(first at {np.argwhere(unexplained)[:4].tolist()})")
    return int(diff.sum()), int((diff & near).sum())


def topp_on_scores(scores: np.ndarray, p: float) -> np.ndarray:
    """The oracle's softmax + Top-P + union applied to given band scores
    [..., 2, nb, nb]; returns (mask, c_excl [..., 2, nb, nb])."""
    shp = scores.shape[:-3]
    flat = scores.reshape((-1,) + scores.shape[-3:])
    masks, cx = [], []
    for s in flat:
        k_hi, c_hi = oracle.top_p(oracle.softmax_rows(s[0]), p)
        k_lo, c_lo = oracle.top_p(oracle.softmax_rows(s[1]), p)
        masks.append(k_hi | k_lo)
        cx.append(np.stack([c_hi, c_lo]))
    nb = scores.shape[-1]
    return (np.stack(masks).reshape(shp + (nb, nb)), np.stack(cx).reshape(shp + (2, nb, nb)))


def run_attention(cfg, q, k, v, mask_words: torch.Tensor):
    o = torch.empty_like(q)
    pb.prism_sparse_attn(cfg, q, k, v, mask_words, o)
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    return o


def check_attention_rows(o_gpu: torch.Tensor, q, k, v, mask_bool: np.ndarray, rows, group, scale=None):
    """Compare sampled (b, h, i) query blocks against the oracle with the same mask."""
    ocpu = o_gpu.float().cpu().numpy()
    worst_max, worst_mean = 0.0, 0.0
    for (b, h, i) in rows:
        ref = oracle.sparse_attention_block(q, k, v, mask_bool[b, h, i], b, h, i, group, scale=scale)
        got = ocpu[b, h, i * 128:(i + 1) * 128]
        err = np.abs(got - ref)
        worst_max = max(worst_max, float(err.max()))
        worst_mean = max(worst_mean, float(err.mean()))
    assert worst_max <= ATTN_MAX_ABS, f"max-abs {worst_max:.4g} > {ATTN_MAX_ABS}"
    assert worst_mean <= ATTN_MEAN_ABS, f"mean-abs {worst_mean:.4g} > {ATTN_MEAN_ABS}"
    return worst_max, worst_mean


def oracle_estimate_streamed(q, k, bands, p, heads=None, batch=0):
    """Run the oracle one Q head at a time (bounded host memory at 128K+)."""
    hq, hkv = q.shape[1], k.shape[1]
    g = hq // hkv
    heads = list(range(hq)) if heads is None else heads
    res = {}
    for h in heads:
        kv = h // g
        r = oracle.estimate(q[batch:batch + 1, h:h + 1], k[batch:batch + 1, kv:kv + 1], bands[0], bands[1], p)
        for key in ("tau", "logits", "c_excl", "mask", "keep_hi", "keep_lo"):
            res.setdefault(key, []).append(r[key][0, 0])
    return {key: np.stack(v) for key, v in res.items()}


def density(mask_bool: np.ndarray) -> float:
    nb = mask_bool.shape[-1]
    return float(mask_bool.sum()) / (mask_bool.size / (nb * nb) * nb * (nb + 1) / 2)


__all__ = ["make_cfg", "run_estimate", "check_tau", "check_scores", "check_mask", "topp_on_scores",
           "topp_fixed_point", "check_topp_exact", "check_pooled",
           "run_attention", "check_attention_rows", "oracle_estimate_streamed", "density", "math"]
