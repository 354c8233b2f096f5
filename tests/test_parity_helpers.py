"""The test-side restatement of the GPU's Top-P decision (tests/parity.py,
``topp_fixed_point``) checked on the CPU against the oracle's fp64 Top-P
(paper.rainbus.top review, method step (6)): on random rows whose decisions
are not within 1e-6 of p the two select the same blocks, and on equal weights
the fixed-point rule keeps exactly the first ceil(p n) blocks (the oracle's
stable order, lower block first)."""
import numpy as np
import pytest

import oracle
from tests import parity as P


def _rows(rng, nb, spread):
    """Causal rows of fp32 weights in (0, 1] with the row maximum at 1."""
    w = np.full((nb, nb), np.nan)
    for i in range(nb):
        x = rng.normal(0.0, spread, i + 1)
        e = np.exp2((x - x.max()) * np.log2(np.e)).astype(np.float32).astype(np.float64)
        e[np.argmax(x)] = 1.0
        w[i, :i + 1] = e
    return w


@pytest.mark.parametrize("spread,p", [(0.3, 0.95), (2.0, 0.9), (5.0, 0.5), (0.01, 0.93)])
def test_fixed_point_rule_matches_oracle_top_p(spread, p):
    rng = np.random.default_rng(int(spread * 100) + int(p * 100))
    nb = 70
    w = _rows(rng, nb, spread)
    keep = P.topp_fixed_point(w[None], p)[0]
    probs = np.where(np.isfinite(w), w, 0.0)
    probs = probs / probs.sum(axis=1, keepdims=True)
    ref_keep, c_excl = oracle.top_p(probs, p)
    decided = np.abs(c_excl - p) > 1e-6
    assert np.array_equal(keep & decided, ref_keep & decided)
    assert keep[np.tril(np.ones((nb, nb), dtype=bool))].sum() > 0


def test_fixed_point_rule_on_equal_weights_keeps_the_first_blocks():
    nb, p = 40, 0.91
    w = np.where(np.tril(np.ones((nb, nb), dtype=bool)), 1.0, np.nan)
    keep = P.topp_fixed_point(w[None], p)[0]
    for i in range(nb):
        k = int(np.ceil(p * (i + 1) - 1e-9))
        assert keep[i, :k].all() and not keep[i, k:].any(), i


def test_fixed_point_rule_keeps_the_crossing_block():
    """Masses 0.6, 0.3, 0.1 (of Z) at p = 0.9: the second block's mass ahead is
    0.6 < 0.9 (kept), the third's is 0.9, not < 0.9 (dropped)."""
    w = np.full((3, 3), np.nan)
    w[2] = [1.0, 0.5, 1.0 / 6.0]
    w[0, 0] = 1.0
    w[1, :2] = [1.0, 1.0]
    keep = P.topp_fixed_point(w[None], 0.9)[0]
    assert keep[2].tolist() == [True, True, False]
    assert keep[1].tolist() == [True, True, False]  # 0.5 ahead < 0.9
