import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def has_gpu():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(autouse=True)
def _default_dtype_guard():
    """Tests must not leak a changed torch default dtype into later tests (buffers handed to
    the C ABI are typed explicitly, but a float64 default once turned an fp32 output buffer
    into a float64 one)."""
    import torch
    before = torch.get_default_dtype()
    yield
    torch.set_default_dtype(before)
