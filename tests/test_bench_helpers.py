"""Host-side helpers of bench.py (no GPU)."""
import numpy as np

import bench
import oracle


def test_causal_mask_words_keep_every_causal_block():
    # the dense reference of the bench keeps every block j <= i, in the ABI's
    # bit layout (word j // 32, bit j % 32), nothing above the diagonal
    for nb in (1, 31, 32, 33, 100, 257):
        words = (nb + 31) // 32
        got = bench.causal_mask_words(nb, words).numpy().view(np.uint32)
        ref = oracle.pack_mask(np.tril(np.ones((1, 1, nb, nb), dtype=bool)))[0, 0]
        assert got.shape == (nb, words)
        assert np.array_equal(got, ref), nb


def test_job_value_is_per_layer_over_ranks():
    assert bench.job_value(12.0, 4) == 3.0
