import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size case, minutes of CPU")


@pytest.fixture(scope="session")
def cuda_lib():
    """The loaded C-ABI library on a GPU machine; GPU tests depend on it and fail
    loudly (rather than skip) when it cannot be loaded."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected on a machine without CUDA; run with -m 'not gpu'")
    import w4a4_hadamard_rotated_b200 as w4
    w4.load_library()
    return w4
