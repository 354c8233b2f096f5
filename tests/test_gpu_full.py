"""Full-size workloads in the launch configuration bench.py times
(prism_prefill, workspace, mask out), checked on samples the oracle can
compute one by one, plus properties that hold at any size.  Every length of
the long-context sweep (8K, 16K, 64K, 128K, 256K) is checked.

Sampling: the estimator oracle runs on 4 Q heads (one from each of 4 KV
groups, the seed picks the head within the group); the attention oracle on
those heads x query blocks {0, 1, nb/2, nb-1} and two seeded random blocks.
"""
import zlib

import numpy as np
import pytest
import torch

import block_sparse_attention_band_b200 as pb
import oracle
from tests import gen
from tests import parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["llama3_8b_32k", "llama3_8b_128k", "qwen3_8b_64k_planted",
        "sweep_8k", "sweep_16k", "sweep_64k", "sweep_128k", "sweep_256k"]


def _sample_heads(w, rng):
    g = w.hq // w.hkv
    groups = sorted(rng.choice(w.hkv, min(4, w.hkv), replace=False).tolist())
    return [kv * g + int(rng.integers(g)) for kv in groups]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_parity(name, cuda_device):
    w = gen.WORKLOADS[name]
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    q, k, v = gen.make_inputs(w)
    qd, kd, vd = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    cfg = P.make_cfg(w)
    nb, W = w.nb, cfg.words
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=cuda_device)
    mask = torch.empty(w.batch, w.hq, nb, W, dtype=torch.int32, device=cuda_device)
    o = torch.empty_like(qd)
    pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws)
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    words = mask.cpu().numpy().view(np.uint32)

    # properties at full size: causal, >= 1 block per row, finite output
    mb = oracle.unpack_mask(words, nb)
    assert not np.any(mb & ~np.tril(np.ones((nb, nb), dtype=bool)))
    assert np.all(mb.sum(-1) >= 1)
    assert torch.isfinite(o.float()).all()

    # scores / tau on sampled heads (same estimator launch, debug outputs on)
    heads = _sample_heads(w, rng)
    tri = nb * (nb + 1) // 2
    scores = torch.empty(w.batch, w.hq, 2, tri, dtype=torch.float32, device=cuda_device)
    weights = torch.empty(w.batch, w.hq, 2, tri, dtype=torch.float32, device=cuda_device)
    tau = torch.empty(w.batch, w.hq, 2, dtype=torch.float32, device=cuda_device)
    pooled = torch.empty(w.batch * (w.hq + w.hkv), nb, 128, dtype=torch.float32, device=cuda_device)
    mask2 = torch.empty_like(mask)
    pb.prism_estimate(cfg, qd, kd, mask2, ws, dbg_scores=scores, dbg_tau=tau, dbg_weights=weights,
                      dbg_pooled=pooled)
    torch.cuda.synchronize()
    assert torch.equal(mask2, mask), "estimate and prefill disagree on the mask"
    # pooled means of the sampled Q heads and their KV heads, element by element
    g = w.hq // w.hkv
    prow = heads + sorted({w.hq + h // g for h in heads})
    P.check_pooled(pooled[prow].cpu().double().numpy(), q, k, only=prow)
    del pooled
    # Top-P of the sampled heads restated in fixed point on the GPU's own weights: bit-exact
    wt = P.unpack_tri(weights[0, heads].cpu().double().numpy(), nb)
    wt[~np.isfinite(wt)] = np.nan
    P.check_topp_exact(mb[0, heads], wt, w.p)
    del weights, wt
    # the prefill's attention starts while its estimator still runs: every
    # output row must equal a separate attention call on the final mask
    o_sep = torch.empty_like(o)
    pb.prism_sparse_attn(cfg, qd, kd, vd, mask, o_sep)
    torch.cuda.synchronize()
    assert torch.equal(o_sep, o), "overlapped prefill differs from separate calls"
    del o_sep
    hi, lo = gen.default_bands()
    ref = P.oracle_estimate_streamed(q, k, (hi, lo), w.p, heads=heads)
    sc = P.unpack_tri(scores[0, heads].cpu().double().numpy(), nb)
    P.check_tau(tau[0, heads].cpu().double().numpy(), ref)
    P.check_scores(sc, ref)
    n_diff, n_exempt = P.check_mask(mb[0, heads], ref, w.p)
    n_window = int(sum((np.abs(ref["c_excl"][:, z] - w.p) < P.MASK_WINDOW).sum() for z in range(2)))
    print(f"{name}: density {P.density(mb):.4f}, sampled-head mask mismatches {n_diff} (all exempt: {n_exempt}; "
          f"blocks in the 1e-4 window: {n_window})")

    # attention on sampled (head, query block) rows with the GPU's mask
    blocks = sorted({0, 1, nb // 2, nb - 1} | set(rng.integers(0, nb, 2).tolist()))
    rows = [(0, h, i) for h in heads for i in blocks]
    worst = P.check_attention_rows(o, q, k, v, mb, rows, w.hq // w.hkv)
    print(f"{name}: attention rows {len(rows)}, max-abs {worst[0]:.3g}, mean-abs {worst[1]:.3g}")
