"""fp64 CPU oracle for Prism's estimator and block-sparse causal attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.
"""
from .prism_oracle import *  # noqa: F401,F403
from .prism_oracle import (band_logits, band_slice, dense_causal_attention, estimate,
                           estimate_head, mean_pool, pack_mask, rms, softmax_rows,
                           sparse_attention_block, tau_rms, to_f64, top_p, unpack_mask)
