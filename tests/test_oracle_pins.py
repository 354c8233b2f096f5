"""Pins for the fp64 oracle, against what the pages and the mathematics fix.

None of these tests touches the CUDA path.  Each pin is chosen so that a
plausible slip in the oracle (a dropped scale factor, swapped bands, a
transposed product, an off-by-one in the Top-P scan, a wrong GQA mapping)
fails at least one of them.  Page citations: "Prism: Spectral-Aware
Block-Sparse Attention" -- paper.rainbus.top review (method steps (1)-(7),
novelty paragraph), gist.science Technical Summary (sections 1, 2A, 2B).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from tests import gen


# ----------------------------------------------------------------------------
# pooling: closed forms (review: novelty paragraph, lambda_j(B) ~ sinc(B theta_j / 2 pi))
# ----------------------------------------------------------------------------
def test_pool_constant_and_ramp():
    rng = np.random.default_rng(0)
    c = rng.standard_normal(7)
    x = np.tile(c, (12, 1))  # 12 tokens, constant
    np.testing.assert_allclose(oracle.mean_pool(x, 4), np.tile(c, (3, 1)), rtol=0, atol=1e-15)
    t = np.arange(12, dtype=np.float64)[:, None] * np.ones((1, 3))
    pooled = oracle.mean_pool(t, 4)
    # mean of t0..t0+3 is the midpoint t0 + 1.5
    np.testing.assert_allclose(pooled[:, 0], [1.5, 5.5, 9.5], rtol=0, atol=1e-15)


def test_pool_short_last_block():
    """A sequence that is not a multiple of the block: the last block is the
    mean over its own tokens (constant -> the constant, ramp -> its midpoint)."""
    c = np.array([0.5, -2.0, 3.25])
    x = np.tile(c, (11, 1))  # 11 tokens, blocks of 4: 4 + 4 + 3
    np.testing.assert_allclose(oracle.mean_pool(x, 4), np.tile(c, (3, 1)), rtol=0, atol=1e-15)
    t = np.arange(11, dtype=np.float64)[:, None] * np.ones((1, 2))
    pooled = oracle.mean_pool(t, 4)
    np.testing.assert_allclose(pooled[:, 0], [1.5, 5.5, 9.0], rtol=0, atol=1e-15)
    # the exact case still agrees with the reshape definition
    np.testing.assert_allclose(oracle.mean_pool(t[:8], 4)[:, 0], [1.5, 5.5], rtol=0, atol=0)


def test_short_last_block_attention_is_dense_on_valid_tokens():
    """Attention of the short last query block over all kept blocks equals
    plain causal attention of those tokens over the whole (short) sequence."""
    rng = np.random.default_rng(5)
    n, d = 2 * 16 + 5, 8
    q = rng.standard_normal((1, 1, n, d))
    k = rng.standard_normal((1, 1, n, d))
    v = rng.standard_normal((1, 1, n, d))
    full = np.ones(3, dtype=bool)
    got = oracle.sparse_attention_block(q, k, v, full, 0, 0, 2, 1, block=16)
    s = q[0, 0] @ k[0, 0].T / np.sqrt(d)
    s = np.where(np.tril(np.ones((n, n), dtype=bool)), s, -np.inf)
    pr = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (pr / pr.sum(axis=1, keepdims=True)) @ v[0, 0]
    assert got.shape == (5, d)
    np.testing.assert_allclose(got, ref[32:], rtol=1e-12, atol=1e-12)


def test_pool_matches_library_avg_pool():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 256, 16))
    ref = torch.nn.functional.avg_pool1d(torch.from_numpy(x).transpose(1, 2), 64).transpose(1, 2)
    np.testing.assert_allclose(oracle.mean_pool(x, 64), ref.numpy(), rtol=1e-14, atol=1e-14)


def _dirichlet(theta, block):
    # |(1/B) sum_{t<B} exp(i t theta)| summed as a geometric series
    return np.abs(np.sin(block * theta / 2.0) / (block * np.sin(theta / 2.0)))


@pytest.mark.parametrize("base,dead_last", [(5e5, 14), (1e6, 13)])
@pytest.mark.parametrize("t0", [0, 128 * 37])
def test_pooled_rope_attenuation_closed_form(base, dead_last, t0):
    """A constant pre-RoPE vector, rotated at B consecutive positions and mean
    pooled, keeps a fraction lambda_j of each pair's magnitude: exactly the
    Dirichlet kernel, approximately the normalised sinc the review prints."""
    B, D = 128, 128
    rng = np.random.default_rng(2)
    c = torch.from_numpy(rng.standard_normal(D))
    cos, sin = gen.rope_tables(B, D, base, start=t0)
    x = gen.apply_rope(c[None, :].expand(B, D).clone(), cos, sin).numpy()
    pooled = oracle.mean_pool(x, B)[0]
    half = D // 2
    pair_in = np.hypot(c.numpy()[:half], c.numpy()[half:])
    pair_out = np.hypot(pooled[:half], pooled[half:])
    lam = pair_out / pair_in
    theta = np.array(gen.rope_theta(D, base))
    np.testing.assert_allclose(lam, _dirichlet(theta, B), rtol=0, atol=1e-12)
    sinc = np.abs(np.sinc(B * theta / (2 * np.pi)))  # np.sinc is sin(pi x)/(pi x)
    assert np.max(np.abs(lam - sinc)) < 6.2e-4
    assert np.max(np.abs(lam[16:] - sinc[16:])) < 1.9e-5
    # dead zone: B theta_j >= 2 pi exactly for j <= dead_last; there lambda stays
    # under the first side-lobe peak of |sinc| (0.2172...), pair 0 nearly vanishes
    assert np.all(B * theta[: dead_last + 1] >= 2 * np.pi)
    assert B * theta[dead_last + 1] < 2 * np.pi
    assert np.all(lam[: dead_last + 1] < 0.2173 + 6.2e-4)
    assert abs(lam[0] - 0.014992324865) < 1e-9
    # semantic zone (the slow pairs the low band holds) passes almost unattenuated
    assert np.all(lam[32:] > 0.99)


# ----------------------------------------------------------------------------
# a worked example derived by hand from steps (2)-(7)
# ----------------------------------------------------------------------------
# D = 2, B = 2, N = 4, high band = {dim 0}, low band = {dim 1} (d_z = 1).
HAND_Q = np.array([[1, 0], [1, 0], [2, 2], [0, 2]], dtype=np.float64)  # Qbar = [1,0],[1,2]
HAND_K = np.array([[3, 1], [1, 1], [0, 4], [0, 0]], dtype=np.float64)  # Kbar = [2,1],[0,2]


def _hand_estimate(p, tau_mode, tau_explicit=(1.0, 1.0)):
    q = HAND_Q[None, None]
    k = HAND_K[None, None]
    return oracle.estimate(q, k, [0], [1], p, block=2, tau_mode=tau_mode, tau_explicit=tau_explicit)


def test_hand_example_rms_temperature():
    r = _hand_estimate(0.8, "rms")
    # RMS of pooled bands: Q hi [1,1] -> 1, Q lo [0,2] -> sqrt 2, Q full -> sqrt(6/4);
    # K hi [2,0] -> sqrt 2, K lo [1,2] -> sqrt(5/2), K full -> sqrt(9/4) = 1.5
    np.testing.assert_allclose(r["rms_q"][0, 0], [1.0, math.sqrt(2), math.sqrt(1.5)], rtol=1e-15)
    np.testing.assert_allclose(r["rms_k"][0, 0], [math.sqrt(2), math.sqrt(2.5), 1.5], rtol=1e-15)
    den = math.sqrt(1.5) * 1.5
    tau_hi = 1.0 * math.sqrt(2) / den
    tau_lo = math.sqrt(2) * math.sqrt(2.5) / den
    np.testing.assert_allclose(r["tau"][0, 0], [tau_hi, tau_lo], rtol=1e-14)
    lg = r["logits"][0, 0]
    # hi: Qbar_hi[i] * Kbar_hi[j] / (tau_hi * sqrt 1): rows (1*2, -), (1*2, 1*0)
    np.testing.assert_allclose(lg[0, 0, 0], 2 / tau_hi, rtol=1e-14)
    np.testing.assert_allclose(lg[0, 1, :], [2 / tau_hi, 0.0], rtol=1e-14, atol=1e-15)
    # lo: rows (0*1, -), (2*1, 2*2)
    np.testing.assert_allclose(lg[1, 1, :], [2 / tau_lo, 4 / tau_lo], rtol=1e-14)
    assert lg[0, 0, 1] == -np.inf and lg[1, 0, 1] == -np.inf
    ph = 1.0 / (1.0 + math.exp(-2 / tau_hi))          # hi row 1: P(j=0)
    pl = 1.0 / (1.0 + math.exp(2 / tau_lo))           # lo row 1: P(j=0)
    np.testing.assert_allclose(r["probs"][0, 0, 0, 1], [ph, 1 - ph], rtol=1e-13)
    np.testing.assert_allclose(r["probs"][0, 0, 1, 1], [pl, 1 - pl], rtol=1e-13)
    # p = 0.8: hi keeps only j=0 (0.93 >= 0.8), lo keeps only j=1 (0.84 >= 0.8)
    assert ph > 0.8 and 1 - pl > 0.8
    np.testing.assert_array_equal(r["keep_hi"][0, 0], [[True, False], [True, False]])
    np.testing.assert_array_equal(r["keep_lo"][0, 0], [[True, False], [False, True]])
    np.testing.assert_array_equal(r["mask"][0, 0], [[True, False], [True, True]])


def test_hand_example_explicit_temperature():
    r = _hand_estimate(0.95, "explicit", (0.5, 2.0))
    lg = r["logits"][0, 0]
    np.testing.assert_allclose(lg[0, 1], [4.0, 0.0], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(lg[1, 1], [1.0, 2.0], rtol=1e-15)
    e4 = math.exp(4.0)
    np.testing.assert_allclose(r["probs"][0, 0, 0, 1], [e4 / (e4 + 1), 1 / (e4 + 1)], rtol=1e-14)
    np.testing.assert_allclose(r["probs"][0, 0, 1, 1], [1 / (1 + math.e), math.e / (1 + math.e)],
                               rtol=1e-14)
    # hi row 1: 0.982 >= 0.95 -> {0};  lo row 1: 0.731 < 0.95 -> both kept
    np.testing.assert_array_equal(r["keep_hi"][0, 0][1], [True, False])
    np.testing.assert_array_equal(r["keep_lo"][0, 0][1], [True, True])
    # c_excl of the dropped hi block is the mass ahead of it
    np.testing.assert_allclose(r["c_excl"][0, 0, 0, 1, 1], e4 / (e4 + 1), rtol=1e-14)


# ----------------------------------------------------------------------------
# temperature invariants (review step 4; summary 2B)
# ----------------------------------------------------------------------------
def _small_inputs(seed=5, hq=2, hkv=1, n=1024):
    w = gen.small_workload("pin", 1, hq, hkv, n, seed)
    q, k, _ = gen.make_inputs(w, with_v=False)
    return q.double().numpy(), k.double().numpy()


def test_tau_scale_invariance_and_full_band():
    q, k = _small_inputs()
    hi, lo = gen.default_bands()
    r1 = oracle.estimate(q, k, hi, lo, 0.9)
    r2 = oracle.estimate(3.0 * q, 0.25 * k, hi, lo, 0.9)
    np.testing.assert_allclose(r1["tau"], r2["tau"], rtol=1e-13)
    # logits scale with the product of the factors, probabilities do not stay
    np.testing.assert_allclose(r2["logits"][np.isfinite(r2["logits"])],
                               0.75 * r1["logits"][np.isfinite(r1["logits"])], rtol=1e-12)
    full = list(range(128))
    r3 = oracle.estimate(q, k, full, full, 0.9)
    np.testing.assert_allclose(r3["tau"], 1.0, rtol=1e-14)
    # the attenuated high band gets tau < 1 (its logits are boosted), the low band ~ 1
    assert np.all(r1["tau"][..., 0] < 1.0)


def test_full_band_explicit_tau_is_plain_pooled_attention():
    """tau = 1 and both bands = all dims: the estimator's scores reduce to plain
    mean-pooled block attention, here built from library routines."""
    q, k = _small_inputs(seed=6, hq=2, hkv=1, n=1024)
    full = list(range(128))
    r = oracle.estimate(q, k, full, full, 0.9, tau_mode="explicit", tau_explicit=(1.0, 1.0))
    qt = torch.from_numpy(q[0])
    kt = torch.from_numpy(k[0])
    qp = torch.nn.functional.avg_pool1d(qt.transpose(1, 2), 128).transpose(1, 2)
    kp = torch.nn.functional.avg_pool1d(kt.transpose(1, 2), 128).transpose(1, 2)
    nb = qp.shape[1]
    causal = torch.ones(nb, nb, dtype=torch.bool).tril()
    for h in range(2):
        s = (qp[h] @ kp[0].T) / math.sqrt(128)
        prob = torch.softmax(s.masked_fill(~causal, float("-inf")), dim=-1)
        np.testing.assert_allclose(r["probs"][0, h, 0], prob.numpy(), rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(r["probs"][0, h, 1], prob.numpy(), rtol=1e-11, atol=1e-14)


def test_band_choice_matters():
    """Swapping the band sets changes the scores: catches swapped hi / lo."""
    q, k = _small_inputs(seed=7)
    hi, lo = gen.default_bands()
    r = oracle.estimate(q, k, hi, lo, 0.9)
    s = oracle.estimate(q, k, lo, hi, 0.9)
    np.testing.assert_allclose(r["logits"][:, :, 0][np.isfinite(r["logits"][:, :, 0])],
                               s["logits"][:, :, 1][np.isfinite(s["logits"][:, :, 1])], rtol=1e-13)
    assert not np.allclose(r["logits"][:, :, 0][np.isfinite(r["logits"][:, :, 0])],
                           r["logits"][:, :, 1][np.isfinite(r["logits"][:, :, 1])])


def test_batch_elements_are_independent_problems():
    """Each batch element is estimated on its own: a batch of two equals the
    two single-element runs (temperatures, logits, masks), and a change to
    one element leaves the other's results untouched."""
    w = gen.small_workload("batch_pin", 2, 2, 1, 6 * 128, seed=13)
    q, k, _ = gen.make_inputs(w, with_v=False)
    q, k = q.double().numpy(), k.double().numpy()
    hi, lo = gen.default_bands()
    both = oracle.estimate(q, k, hi, lo, 0.9)
    for b in range(2):
        one = oracle.estimate(q[b:b + 1], k[b:b + 1], hi, lo, 0.9)
        np.testing.assert_array_equal(both["tau"][b], one["tau"][0])
        np.testing.assert_array_equal(both["mask"][b], one["mask"][0])
    q2 = q.copy()
    q2[1] *= -1.0
    other = oracle.estimate(q2, k, hi, lo, 0.9)
    np.testing.assert_array_equal(other["mask"][0], both["mask"][0])
    assert not np.array_equal(other["mask"][1], both["mask"][1])


def test_gqa_mapping_equals_repeated_kv_heads():
    """Q head h reads KV head h // (hq / hkv): with every KV head repeated for
    its group, the same problem as multi-head attention (one KV head per Q
    head) gives identical temperatures, logits and masks.  A mapping by
    h % hkv would pair heads differently and fail."""
    w = gen.small_workload("gqa_pin", 1, 4, 2, 8 * 128, seed=12)
    q, k, _ = gen.make_inputs(w, with_v=False)
    q, k = q.double().numpy(), k.double().numpy()
    hi, lo = gen.default_bands()
    g = oracle.estimate(q, k, hi, lo, 0.9)
    m = oracle.estimate(q, np.repeat(k, 2, axis=1), hi, lo, 0.9)
    np.testing.assert_array_equal(g["tau"], m["tau"])
    f = np.isfinite(g["logits"])
    np.testing.assert_array_equal(g["logits"][f], m["logits"][f])
    np.testing.assert_array_equal(g["mask"], m["mask"])
    # and it is not the same as pairing Q head h with KV head h % hkv
    swapped = np.stack([k[:, 0], k[:, 1], k[:, 0], k[:, 1]], axis=1)
    s_ = oracle.estimate(q, swapped, hi, lo, 0.9)
    assert not np.allclose(g["tau"], s_["tau"])


# ----------------------------------------------------------------------------
# softmax rows
# ----------------------------------------------------------------------------
def test_softmax_rows_sum_and_causal():
    q, k = _small_inputs(seed=8)
    hi, lo = gen.default_bands()
    r = oracle.estimate(q, k, hi, lo, 0.95)
    pr = r["probs"]
    np.testing.assert_allclose(pr.sum(-1), 1.0, rtol=0, atol=1e-13)
    nb = pr.shape[-1]
    assert np.all(pr[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] == 0)


# ----------------------------------------------------------------------------
# Top-P (review step 6): brute force on tiny rows
# ----------------------------------------------------------------------------
def _brute_force_top_p(prob, p):
    n = len(prob)
    best = None
    for m in range(1, n + 1):
        sets = [s for s in itertools.combinations(range(n), m) if sum(prob[j] for j in s) >= p]
        if sets:
            best_mass = max(sum(prob[j] for j in s) for s in sets)
            best = (m, best_mass)
            break
    return best


def _row_probs(rng, n, ties=False):
    if ties:
        vals = rng.choice([1.0, 2.0, 4.0], size=n)
    else:
        vals = rng.gamma(0.5, size=n)
    return vals / vals.sum()


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 12])
@pytest.mark.parametrize("ties", [False, True])
def test_top_p_brute_force(n, ties):
    rng = np.random.default_rng(100 + n + 50 * ties)
    for trial in range(20):
        prob = _row_probs(rng, n, ties)
        p = float(rng.uniform(0.3, 0.99))
        # embed the row as the last row of an n x n causal block matrix
        mat = np.zeros((n, n))
        for i in range(n):
            mat[i, : i + 1] = 1.0 / (i + 1)
        mat[n - 1] = prob
        keep, c_excl = oracle.top_p(mat, p)
        kept = np.flatnonzero(keep[n - 1])
        m, best_mass = _brute_force_top_p(prob, p)
        assert len(kept) == m
        assert abs(prob[kept].sum() - best_mass) < 1e-12
        # deterministic tie-break: the kept set is the first m of the order (-prob, j)
        order = sorted(range(n), key=lambda j: (-prob[j], j))
        assert sorted(order[:m]) == list(kept)
        # dropping the lowest-ranked kept block takes the mass below p
        assert prob[kept].sum() >= p - 1e-12
        assert prob[order[: m - 1]].sum() < p


def test_top_p_ties_lower_index_first():
    mat = np.array([[1.0, 0, 0, 0], [0.5, 0.5, 0, 0], [1 / 3, 1 / 3, 1 / 3, 0],
                    [0.25, 0.25, 0.25, 0.25]])
    keep, _ = oracle.top_p(mat, 0.5)
    np.testing.assert_array_equal(keep[3], [True, True, False, False])
    np.testing.assert_array_equal(keep[1], [True, False, False, False])
    np.testing.assert_array_equal(keep[2], [True, True, False, False])


def test_top_p_p1_keeps_all_and_monotone():
    q, k = _small_inputs(seed=9)
    hi, lo = gen.default_bands()
    r1 = oracle.estimate(q, k, hi, lo, 1.0)
    nb = r1["mask"].shape[-1]
    assert np.all(r1["mask"] == np.tril(np.ones((nb, nb), dtype=bool)))
    prev = None
    for p in (0.5, 0.8, 0.9, 0.95, 0.99):
        r = oracle.estimate(q, k, hi, lo, p)
        for key in ("keep_hi", "keep_lo", "mask"):
            assert not np.any(r[key] & ~r1[key])
        if prev is not None:
            for key in ("keep_hi", "keep_lo"):
                assert not np.any(prev[key] & ~r[key])  # monotone in p
        prev = r


def test_top_p_p1_keeps_blocks_of_zero_probability():
    """p >= 1 keeps every causal block even where the mass ahead of a block
    already rounds to 1 (probabilities that underflow to 0): the rule is
    stated for p, not left to the floating-point sum reaching 1."""
    mat = np.array([[1.0, 0, 0], [1.0, 0.0, 0], [1.0, 0.0, 0.0]])
    keep, c_excl = oracle.top_p(mat, 1.0)
    np.testing.assert_array_equal(keep, np.tril(np.ones((3, 3), dtype=bool)))
    assert c_excl[2, 1] == 1.0 and c_excl[2, 2] == 1.0
    # the same through the estimator: a temperature small enough that every
    # row's softmax puts all its mass on one block
    rng = np.random.default_rng(21)
    q = rng.standard_normal((1, 1, 8 * 16, 128))
    k = rng.standard_normal((1, 1, 8 * 16, 128))
    r = oracle.estimate(q, k, list(range(64)), list(range(32, 128)), 1.0, block=16,
                        tau_mode="explicit", tau_explicit=(1e-4, 1e-4))
    assert np.any(r["probs"][0, 0][:, np.tril(np.ones((8, 8), dtype=bool))] == 0.0)
    np.testing.assert_array_equal(r["mask"][0, 0], np.tril(np.ones((8, 8), dtype=bool)))


def test_zero_queries_give_unit_tau_and_uniform_rows():
    """A head whose queries are all zero: every pooled RMS of Q is 0, so both
    temperatures fall back to 1, every causal logit is 0, each row's softmax is
    uniform over its i + 1 blocks, and Top-P (ties to the lower block index)
    keeps exactly the first ceil(p (i + 1)) blocks."""
    rng = np.random.default_rng(22)
    nb, p = 12, 0.61  # p (i + 1) is never within 0.01 of an integer for i < 12
    q = np.zeros((1, 1, nb * 16, 128))
    k = rng.standard_normal((1, 1, nb * 16, 128))
    r = oracle.estimate(q, k, list(range(64)), list(range(32, 128)), p, block=16)
    np.testing.assert_array_equal(r["tau"][0, 0], [1.0, 1.0])
    causal = np.tril(np.ones((nb, nb), dtype=bool))
    for z in range(2):
        np.testing.assert_array_equal(r["logits"][0, 0, z][causal], 0.0)
        np.testing.assert_allclose(r["probs"][0, 0, z], causal / np.arange(1, nb + 1)[:, None],
                                   rtol=1e-15, atol=0)
    want = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        want[i, :math.ceil(p * (i + 1))] = True
    for key in ("keep_hi", "keep_lo", "mask"):
        np.testing.assert_array_equal(r[key][0, 0], want)


def test_union_identities():
    q, k = _small_inputs(seed=10)
    hi, lo = gen.default_bands()
    r = oracle.estimate(q, k, hi, lo, 0.9)
    m, mh, ml = r["mask"], r["keep_hi"], r["keep_lo"]
    assert np.all(m >= mh) and np.all(m >= ml)
    assert m.sum() == mh.sum() + ml.sum() - (mh & ml).sum()
    nb = m.shape[-1]
    assert not np.any(m[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]])
    assert np.all(m.sum(-1) >= 1)  # every row keeps at least one block


# ----------------------------------------------------------------------------
# mask packing
# ----------------------------------------------------------------------------
def test_pack_mask_bit_order():
    m = np.zeros((1, 40), dtype=bool)
    m[0, [0, 2, 33]] = True
    w = oracle.pack_mask(m)
    assert w.shape == (1, 2) and w[0, 0] == 5 and w[0, 1] == 2
    rng = np.random.default_rng(3)
    big = rng.random((3, 70, 70)) < 0.4
    np.testing.assert_array_equal(oracle.unpack_mask(oracle.pack_mask(big), 70), big)


# ----------------------------------------------------------------------------
# attention: p = 1 -> dense causal; arbitrary masks -> library SDPA with the
# equivalent token mask; GQA mapping h -> h // (Hq / Hkv)
# ----------------------------------------------------------------------------
def _sdpa_ref(q, k, v, token_mask, group):
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(k).repeat_interleave(group, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(group, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=token_mask)


def _attn_inputs(seed, hq, hkv, n):
    w = gen.small_workload("pin_attn", 1, hq, hkv, n, seed)
    q, k, v = gen.make_inputs(w)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


def test_attention_dense_causal_vs_library():
    q, k, v = _attn_inputs(11, 4, 2, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k).repeat_interleave(2, dim=1),
        torch.from_numpy(v).repeat_interleave(2, dim=1), is_causal=True).numpy()
    dense = oracle.dense_causal_attention(q, k, v, group=2)
    np.testing.assert_allclose(dense, ref, rtol=1e-10, atol=1e-12)
    nb = 4
    full_mask = np.tril(np.ones((nb, nb), dtype=bool))
    for h in range(4):
        for i in range(nb):
            o = oracle.sparse_attention_block(q, k, v, full_mask[i], 0, h, i, group=2)
            np.testing.assert_allclose(o, ref[0, h, i * 128:(i + 1) * 128], rtol=1e-10, atol=1e-12)


def test_attention_sparse_mask_vs_library():
    q, k, v = _attn_inputs(12, 2, 1, 768)
    nb = 6
    rng = np.random.default_rng(4)
    blk = np.tril(rng.random((nb, nb)) < 0.5)
    blk[np.arange(nb), rng.integers(0, np.arange(nb) + 1)] = True  # >= 1 block per row
    tok = np.repeat(np.repeat(blk, 128, axis=0), 128, axis=1) & np.tril(np.ones((768, 768), dtype=bool))
    ref = _sdpa_ref(q, k, v, torch.from_numpy(tok), 2).numpy()
    for h in range(2):
        for i in range(nb):
            o = oracle.sparse_attention_block(q, k, v, blk[i], 0, h, i, group=2)
            rows_visible = tok[i * 128:(i + 1) * 128].any(axis=1)
            np.testing.assert_allclose(o[rows_visible], ref[0, h, i * 128:(i + 1) * 128][rows_visible],
                                       rtol=1e-10, atol=1e-12)


def test_attention_batch_elements_vs_library():
    """Batch element b reads its own Q, K and V: every element of a batch of two
    matches the library's attention of that element alone (same block mask)."""
    w = gen.small_workload("pin_attn_b2", 2, 2, 1, 512, 14)
    q, k, v = (x.double().numpy() for x in gen.make_inputs(w))
    nb = 4
    rng = np.random.default_rng(6)
    blk = np.tril(rng.random((nb, nb)) < 0.6)
    blk[np.arange(nb), np.arange(nb)] = True
    tok = np.repeat(np.repeat(blk, 128, axis=0), 128, axis=1) & np.tril(np.ones((512, 512), dtype=bool))
    dense = oracle.dense_causal_attention(q, k, v, group=2)
    for b in range(2):
        ref = _sdpa_ref(q[b:b + 1], k[b:b + 1], v[b:b + 1], torch.from_numpy(tok), 2).numpy()
        causal_ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b]), torch.from_numpy(k[b]).repeat_interleave(2, dim=0),
            torch.from_numpy(v[b]).repeat_interleave(2, dim=0), is_causal=True).numpy()
        np.testing.assert_allclose(dense[b], causal_ref, rtol=1e-10, atol=1e-12)
        for h in range(2):
            for i in range(nb):
                o = oracle.sparse_attention_block(q, k, v, blk[i], b, h, i, group=2)
                np.testing.assert_allclose(o, ref[0, h, i * 128:(i + 1) * 128], rtol=1e-10, atol=1e-12)


def test_attention_diagonal_only_is_local_and_empty_is_zero():
    q, k, v = _attn_inputs(13, 1, 1, 256)
    o = oracle.sparse_attention_block(q, k, v, np.array([False, True]), 0, 0, 1, group=1)
    # local causal attention inside block 1, written out with a library softmax
    qb, kb, vb = (torch.from_numpy(x[0, 0, 128:256]) for x in (q, k, v))
    s = (qb @ kb.T) / math.sqrt(128)
    s = s.masked_fill(~torch.ones(128, 128, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(o, (torch.softmax(s, -1) @ vb).numpy(), rtol=1e-10, atol=1e-12)
    z = oracle.sparse_attention_block(q, k, v, np.array([False, False]), 0, 0, 1, group=1)
    assert np.all(z == 0)


def test_forced_blocks_are_added_after_the_union():
    """force_sink / force_diag only add key block 0 / the diagonal to every row
    of the union; everything else is unchanged."""
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 2, 6 * 16, 128))
    k = rng.standard_normal((1, 1, 6 * 16, 128))
    hi, lo = list(range(64)), list(range(32, 128))
    base = oracle.estimate(q, k, hi, lo, 0.5, block=16)["mask"]
    forced = oracle.estimate(q, k, hi, lo, 0.5, block=16, force_sink=True, force_diag=True)["mask"]
    nb = 6
    extra = np.zeros((nb, nb), dtype=bool)
    extra[:, 0] = True
    extra[np.arange(nb), np.arange(nb)] = True
    np.testing.assert_array_equal(forced, base | extra)
