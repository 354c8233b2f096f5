import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library():
    """Builds libprism_b200.so before any test module imports the package
    (the package refuses to import without it). build.py is loaded by path for
    the same reason."""
    import importlib.util
    path = os.path.join(ROOT, "block_sparse_attention_band_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_prism_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_build_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("a GPU test ran without a CUDA device: the CUDA path is required")
    return torch.device("cuda:0")
