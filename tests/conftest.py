import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture
def dev_lib():
    """The binding routed to the development build (libsegquant_dev.so: the
    environment switches of the measured alternative kernels and the wait
    hooks) for one test."""
    from post_quantized_linear_b200 import _lib
    with _lib.dev_library() as lib:
        yield lib
