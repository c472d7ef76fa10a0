import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built liblq.so")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN


@pytest.fixture(scope="session")
def cuda_device():
    """The GPU tests' device.  On a machine without a usable GPU this fails
    (it does not skip): GPU tests are only collected with ``-m gpu``."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test run on a machine without CUDA")
    return torch.device("cuda:0")
