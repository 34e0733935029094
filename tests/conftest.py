import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and libaqnf4.so")
    config.addinivalue_line("markers", "slow: full-size workloads")


@pytest.fixture(scope="session")
def book():
    import oracle
    return oracle.codebook()


@pytest.fixture(scope="session")
def cuda():
    """The CUDA device; GPU tests fail (not skip) when the library or device is missing."""
    import torch
    from quantized_lora_setup_b200 import aqnf4
    aqnf4.library()  # raises if libaqnf4.so was not built
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    return torch.device("cuda:0")
