import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def kv_gpu():
    """The CUDA library, built and initialised on cuda:0 (GPU tests only)."""
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from quantized_paged_kv_q4_b200 import build, kvattn

    build.build()
    torch.cuda.set_device(0)
    kvattn.kvattn_init(0)
    assert kvattn.kvattn_device_error() == 0
    yield kvattn
    assert kvattn.kvattn_device_error() == 0, "a kernel recorded a device-side error"
