import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def gpu_lib():
    """The CUDA library through its Python binding; skips nothing: a GPU test
    that cannot load the library fails."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_decode_attention_step_b200 as saga
    saga.load()
    return saga
