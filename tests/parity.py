"""Parity rules between the CUDA path and the fp64 oracle (test code only).

Rules (tolerances from the arithmetic of each step):
* temperatures: relative 1e-4 (fp32 sums of <= 2^15 non-negative partials);
* band scores L_z: |L_gpu - L_ref| <= 1e-3 * max(|L_ref|, 1e-3 * max_row |L_ref|)
  on the causal entries (fp32 dot products of 64..96 pooled dims);
* masks: bit-exact, except blocks whose oracle decision quantity (the mass
  ranked strictly ahead, c_excl) lies within 1e-4 of p -- those are exempt and
  counted.  Top-P re-run by the oracle on the GPU's own scores must agree with
  the GPU mask except within 1e-5 of p (fp32 vs fp64 softmax of equal logits);
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


def run_estimate(cfg: pb.PrismConfig, q: torch.Tensor, k: torch.Tensor, with_scores=True):
    """q, k on the GPU.  Returns (mask bool [b,hq,nb,nb], scores [b,hq,2,nb,nb] or None, tau)."""
    b, hq = q.shape[0], q.shape[1]
    nb, W = cfg.nb, cfg.words
    dev = q.device
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
    mask = torch.full((b, hq, nb, W), 0xDEAD, dtype=torch.int32, device=dev)
    tri = nb * (nb + 1) // 2
    scores = torch.empty(b, hq, 2, tri, dtype=torch.float32, device=dev) if with_scores else None
    tau = torch.empty(b, hq, 2, dtype=torch.float32, device=dev)
    pb.prism_estimate(cfg, q, k, mask, ws, dbg_scores=scores, dbg_tau=tau)
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    words = mask.cpu().numpy().view(np.uint32)
    m = oracle.unpack_mask(words, nb)
    sc = unpack_tri(scores.cpu().double().numpy(), nb) if with_scores else None
    return m, sc, tau.cpu().double().numpy(), words


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
           "run_attention", "check_attention_rows", "oracle_estimate_streamed", "density", "math"]
