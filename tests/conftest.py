import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def _cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda():
    """The CUDA device, or a hard failure: GPU tests never fall back to the CPU."""
    if not _cuda_ok():
        pytest.fail("GPU test selected but no CUDA device is visible")
    import torch
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def bl(cuda):
    """The BitLinear binding over the in-tree CUDA library (fails loudly if missing)."""
    import int8_row_absmax_b200 as pkg
    pkg.load()
    return pkg
