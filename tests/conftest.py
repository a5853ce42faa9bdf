import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def y_tolerance(bound):
    """Acceptance bound on |y_gpu - y_ref| per element: 8e-3 * sum_k |xhat_k * what_k| + 1e-6."""
    return 8e-3 * bound + 1e-6


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
