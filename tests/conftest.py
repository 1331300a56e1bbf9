import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: large CPU case")


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _guard_bands(request):
    """For GPU tests: output buffers allocated through helpers.GUARD sit between sentinel
    guard bands; after the test every guard byte must be unchanged."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    from helpers import GUARD

    GUARD.reset()
    yield
    try:
        GUARD.check()
    finally:
        GUARD.reset()
