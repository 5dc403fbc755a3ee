import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200 / sm_100a); runs the CUDA library")
    config.addinivalue_line("markers", "slow: long CPU test")


@pytest.fixture(autouse=True)
def _gpu_guard(request):
    """GPU tests fail loudly (never skip) when no CUDA device is visible."""
    if request.node.get_closest_marker("gpu") is not None:
        import torch
        if not torch.cuda.is_available():
            pytest.fail("GPU test run without a visible CUDA device")
    yield

