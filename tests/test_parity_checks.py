"""The comparators the GPU parity tests use reject wrong results.

Each check of ``tests/parity.py`` is given, on the CPU, an oracle result
rounded to the precision the kernels write (it must accept it) and the same
result with one mistake planted in it (it must reject it): a pooled mean off
by a few tolerance units, a row of the wrong head, a temperature or a score
just outside its bound, a mask bit flipped where the decision is clear, a bit
above the diagonal, an attention row computed without one of its kept blocks
or from the wrong KV head.  A comparator that passed everything would make the
GPU parity tests vacuous; these cases show that each one has teeth.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import gen
from tests import parity as P


def _pooled_like_gpu(q, k, seq_tokens=None):
    """The pooled means in the kernels' debug layout [b*hq + b*hkv, nb, 128],
    rounded to fp32."""
    b, hq, n, _ = q.shape
    rows = [(q, bi, h) for bi in range(b) for h in range(hq)] + [(k, bi, h) for bi in range(b) for h in range(k.shape[1])]
    nb = -(-n // 128)
    out = np.zeros((len(rows), nb, 128))
    for r, (x, bi, h) in enumerate(rows):
        nt = n if seq_tokens is None else seq_tokens[bi]
        m = oracle.mean_pool(oracle.to_f64(x[bi, h, :nt]), 128)
        out[r, :m.shape[0]] = m.astype(np.float32)
    return out


def test_check_pooled_has_teeth():
    w = gen.small_workload("chk_pool", 1, 4, 2, 6 * 128, seed=31)
    q, k, _ = gen.make_inputs(w, with_v=False)
    good = _pooled_like_gpu(q, k)
    P.check_pooled(good, q, k)
    # one mean off by 4 tolerance units
    scale = oracle.mean_pool(np.abs(oracle.to_f64(q[0, 2])), 128)
    bad = good.copy()
    bad[2, 3, 17] += 4 * P.POOL_REL * scale[3, 17]
    with pytest.raises(AssertionError):
        P.check_pooled(bad, q, k)
    # two Q heads' rows exchanged
    bad = good.copy()
    bad[[0, 1]] = bad[[1, 0]]
    with pytest.raises(AssertionError):
        P.check_pooled(bad, q, k)
    # a short last block divided by the full block size
    lens = [6 * 128 - 50]
    good = _pooled_like_gpu(q, k, seq_tokens=lens)
    P.check_pooled(good, q, k, seq_tokens=lens)
    bad = good.copy()
    bad[:, 5] *= (128 - 50) / 128
    with pytest.raises(AssertionError):
        P.check_pooled(bad, q, k, seq_tokens=lens)


def _estimate_case(p=0.9):
    w = gen.small_workload("chk_est", 1, 2, 1, 12 * 128, seed=32)
    q, k, _ = gen.make_inputs(w, with_v=False)
    hi, lo = gen.default_bands()
    return oracle.estimate(q, k, hi, lo, p)


def test_check_tau_and_scores_have_teeth():
    ref = _estimate_case()
    tau = ref["tau"].astype(np.float32).astype(np.float64)
    P.check_tau(tau, ref)
    with pytest.raises(AssertionError):
        P.check_tau(tau * (1 + 3e-4), ref)
    lg = ref["logits"]
    sc = np.where(np.isfinite(lg), lg.astype(np.float32), -np.inf).astype(np.float64)
    P.check_scores(sc, ref)
    bad = sc.copy()
    bad[0, 1, 0, 7, 3] *= 1 + 3e-3
    with pytest.raises(AssertionError):
        P.check_scores(bad, ref)
    bad = sc.copy()
    bad[0, 0, 1, 9, 9] = -np.inf  # a causal entry missing
    with pytest.raises(AssertionError):
        P.check_scores(bad, ref)


def test_check_mask_has_teeth():
    p = 0.9
    ref = _estimate_case(p)
    mask = ref["mask"].copy()
    assert P.check_mask(mask, ref, p) == (0, 0)
    cx = ref["c_excl"][0]  # [hq, 2, nb, nb]
    nb = mask.shape[-1]
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    clear = causal[None] & np.all(np.abs(cx - p) > 1e-2, axis=1)
    h, i, j = np.argwhere(clear)[len(np.argwhere(clear)) // 2]
    with pytest.raises(AssertionError):
        P.check_mask(_flip(mask, h, i, j), ref, p)
    bad = mask.copy()
    bad[0, 0, 2, 5] = True  # above the diagonal
    with pytest.raises(AssertionError):
        P.check_mask(bad, ref, p)
    # a block whose decision quantity lies within the window of p is exempt and counted
    near = {key: val.copy() for key, val in ref.items()}
    near["c_excl"][0, h, 0, i, j] = p + 0.5 * P.MASK_WINDOW
    assert P.check_mask(_flip(mask, h, i, j), near, p) == (1, 1)


def _flip(mask, h, i, j):
    out = mask.copy()
    out[0, h, i, j] = not out[0, h, i, j]
    return out


def test_check_topp_exact_has_teeth():
    rng = np.random.default_rng(33)
    nb, p = 24, 0.93
    w = np.full((1, 1, 2, nb, nb), np.nan)
    for z in range(2):
        for i in range(nb):
            x = rng.normal(0.0, 1.5, i + 1)
            e = np.exp(x - x.max()).astype(np.float32).astype(np.float64)
            e[np.argmax(x)] = 1.0
            w[0, 0, z, i, :i + 1] = e
    keep = P.topp_fixed_point(w, p)
    mask = keep[:, :, 0] | keep[:, :, 1]
    P.check_topp_exact(mask, w, p)
    i = nb - 1
    j = int(np.flatnonzero(~mask[0, 0, i, :i + 1])[0])
    with pytest.raises(AssertionError):
        P.check_topp_exact(_flip(mask, 0, i, j), w, p)
    forced = mask.copy()
    forced[..., :, 0] = True
    P.check_topp_exact(forced, w, p, force_sink=True)
    if not np.array_equal(forced, mask):
        with pytest.raises(AssertionError):
            P.check_topp_exact(forced, w, p)


def test_check_attention_rows_has_teeth():
    w = gen.small_workload("chk_attn", 1, 4, 2, 5 * 128, seed=34)
    q, k, v = gen.make_inputs(w)
    nb, group = 5, 2
    rng = np.random.default_rng(35)
    blk = np.tril(rng.random((1, 4, nb, nb)) < 0.5)
    blk[..., np.arange(nb), np.arange(nb)] = True
    blk[..., :, 0] = True  # rows i >= 1 keep at least two blocks
    rows = [(0, h, i) for h in range(4) for i in range(nb)]

    def outputs(mask, kk=k, vv=v):
        o = np.zeros(q.shape)
        for (b, h, i) in rows:
            o[b, h, i * 128:(i + 1) * 128] = oracle.sparse_attention_block(q, kk, vv, mask[b, h, i], b, h, i, group)
        return torch.from_numpy(o).to(torch.bfloat16)

    P.check_attention_rows(outputs(blk), q, k, v, blk, rows, group)
    dropped = blk.copy()
    dropped[0, 3, 4, 0] = False  # one kept block left out of one row
    with pytest.raises(AssertionError):
        P.check_attention_rows(outputs(dropped), q, k, v, blk, rows, group)
    # every Q head answered from the other KV head
    with pytest.raises(AssertionError):
        P.check_attention_rows(outputs(blk, k[:, [1, 0]], v[:, [1, 0]]), q, k, v, blk, rows, group)


def test_unpack_tri_row_order():
    """Packed lower-triangular rows are laid out row by row, j ascending."""
    nb = 4
    packed = np.arange(nb * (nb + 1) // 2, dtype=np.float64)
    out = P.unpack_tri(packed, nb)
    assert out[0, 0] == 0 and out[1, 0] == 1 and out[1, 1] == 2 and out[2, 1] == 4 and out[3, 3] == 9
    assert np.all(np.isneginf(out[np.triu_indices(nb, 1)]))
