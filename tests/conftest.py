import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def pytest_collection_modifyitems(config, items):
    # GPU tests never run silently on a machine without a GPU: they are
    # deselected with -m "not gpu" and fail loudly otherwise.
    pass


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()
