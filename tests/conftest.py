import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libq4dec")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch

    # GPU tests run only under ``-m gpu`` on a CUDA box; a missing device or a
    # missing library there is a failure, never a silent skip.
    assert torch.cuda.is_available(), "gpu-marked test needs a CUDA device"
    return True
