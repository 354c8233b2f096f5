"""Seeded random configurations, every output against the fp64 oracle.

Each case draws batch, head counts and GQA group, a length that is usually
not a multiple of the block (1 to 8000 tokens, up to 63 blocks), p
(including the extremes 0.05 and 1), band index sets (the default pairs or
arbitrary subsets) and the
input recipe's options (per-head means, non-stationary segments, planted
stripes), then checks the estimator (pooled block means, tau, scores, the mask
against the oracle and bit for bit against the fixed-point Top-P on the
kernel's own weights) and the attention (every output row against the oracle
with the kernel's mask).  The draws are fixed by the case seed.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import gen
from tests import parity as P

pytestmark = pytest.mark.gpu

N_CASES = 32


def draw_case(seed: int):
    rng = np.random.default_rng(1000 + seed)
    hkv = int(rng.integers(1, 4))
    group = int(rng.choice([1, 2, 3, 4, 8]))
    batch = int(rng.integers(1, 3))
    seqlen = int(rng.integers(1, 8000)) if seed % 4 else int(rng.integers(1, 64)) * 128
    p = float(rng.choice([0.05, 0.3, 0.6, 0.8, 0.9, 0.95, 0.99, 1.0]))
    kw = {}
    if rng.random() < 0.3:
        kw["segment"] = int(rng.choice([256, 512, 1024]))
    if rng.random() < 0.2 and hkv >= 2:
        kw["stripes"] = True
    w = gen.small_workload(f"fuzz{seed}", batch, hkv * group, hkv, seqlen, seed=2000 + seed, p=p,
                           rope_base=float(rng.choice([1e4, 5e5, 1e6])), **kw)
    if rng.random() < 0.5:
        bands = gen.default_bands()
    else:
        bands = (sorted(rng.choice(128, int(rng.integers(1, 129)), replace=False).tolist()),
                 sorted(rng.choice(128, int(rng.integers(1, 129)), replace=False).tolist()))
    return w, bands


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_configuration(seed, cuda_device):
    w, (hi, lo) = draw_case(seed)
    q, k, v = gen.make_inputs(w)
    qd, kd, vd = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    cfg = P.make_cfg(w, bands=(hi, lo))
    ex = {}
    mask, sc, tau, words = P.run_estimate(cfg, qd, kd, extras=ex)
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_pooled(ex["pooled"], q, k)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    n_diff, n_exempt = P.check_mask(mask, ref, w.p)
    if w.p < 1.0:
        P.check_topp_exact(mask, ex["weights"], w.p)
    else:
        causal = np.tril(np.ones((w.nb, w.nb), dtype=bool))
        assert np.array_equal(mask, np.broadcast_to(causal, mask.shape)), "p = 1 keeps every causal block"
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(b, h, i) for b in range(w.batch) for h in range(w.hq) for i in range(w.nb)]
    if len(rows) > 64:
        rows = [rows[x] for x in sorted(np.random.default_rng(seed).choice(len(rows), 64, replace=False))]
    P.check_attention_rows(o, q, k, v, mask, rows, w.hq // w.hkv)
    print(f"{w.name}: b {w.batch} hq {w.hq} hkv {w.hkv} N {w.seqlen} p {w.p} bands {len(hi)}/{len(lo)} "
          f"density {P.density(mask):.3f} mismatches {n_diff} (exempt {n_exempt})")
