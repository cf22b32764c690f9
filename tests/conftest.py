import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")
    config.addinivalue_line("markers", "late: run after the other tests (the newest checks)")


def pytest_collection_modifyitems(config, items):
    """Tests marked `late` run after all others, in their collected order, so that when a run
    stops at its first failure a failure among the newest checks cannot hide the results of the
    established ones."""
    items[:] = [i for i in items if i.get_closest_marker("late") is None] + \
        [i for i in items if i.get_closest_marker("late") is not None]


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
