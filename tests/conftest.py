import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU test")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture
def kernel_flags():
    """Sets the library's kernel-choice flags for one test and restores the
    previous ones afterwards."""
    import long_context_diffusion_b200 as dl
    saved = []

    def set_flags(flags):
        saved.append(dl.dl_set_kernel_flags(flags))

    yield set_flags
    if saved:
        dl.dl_set_kernel_flags(saved[0])
