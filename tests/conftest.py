import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built librtv.so")
    config.addinivalue_line("markers", "slow: long-running parity case")


def cuda_ok() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def gpu():
    """Skip-free guard: a test marked gpu must run on a GPU; fail loudly."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("test marked gpu needs a CUDA device")
    return torch.device("cuda:0")
