import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (a B200) and the built library")
    config.addinivalue_line("markers", "slow: long-running oracle comparison at full model sizes")


@pytest.fixture(scope="session")
def cuda_device():
    """GPU tests fail (they do not skip) when no CUDA device is visible."""
    import torch
    assert torch.cuda.is_available(), "gpu-marked test run without a CUDA device"
    return torch.device("cuda:0")
