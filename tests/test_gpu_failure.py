"""Failure detection without a GPU fault: every wait in the kernels is bounded;
a wait that runs out records PRISM_ERR_TIMEOUT in a device word, the kernel
returns normally, the host reads the status, and the context stays usable."""
import time

import numpy as np
import pytest
import torch

import block_sparse_attention_band_b200 as pb
import oracle
from tests import gen
from tests import parity as P


@pytest.mark.gpu
def test_bounded_waits_give_up_and_report(cuda_device):
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    t0 = time.perf_counter()
    pb.prism_selftest_wait_timeout(50_000)  # two waits of 50 ms on things nothing signals
    status = pb.prism_get_last_device_error()  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == -10, pb.prism_status_str(status)
    assert 0.09 <= elapsed < 10.0
    assert pb.prism_get_last_device_error() == 0  # reading clears it


@pytest.mark.gpu
def test_context_usable_after_a_timeout(cuda_device):
    pb.prism_selftest_wait_timeout(1_000)
    assert pb.prism_get_last_device_error() == -10
    w = gen.small_workload("after_timeout_nb6", 1, 2, 1, 6 * 128, seed=61, p=0.9)
    q, k, v = gen.make_inputs(w)
    cfg = P.make_cfg(w)
    mask, _, _, _ = P.run_estimate(cfg, q.to(cuda_device), k.to(cuda_device), with_scores=False)
    hi, lo = gen.default_bands()
    P.check_mask(mask, oracle.estimate(q, k, hi, lo, w.p), w.p)
    assert pb.prism_get_last_device_error() == 0


def test_selftest_rejects_bad_limits():
    assert pb.lib.prism_selftest_wait_timeout(None, 0) == -2
    assert pb.lib.prism_selftest_wait_timeout(None, 2_000_001) == -2
