import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def y_tolerance(bound, y_ref=None, y_out=None):
    """Acceptance bound on |y_gpu - y_ref| per element: 8e-3 * sum_k |xhat_k * what_k| + 1e-6.

    With y_ref and y_out (float64 arrays) it also admits the rounding of y to
    bf16 that the layer's output format imposes: half a bf16 ulp of the larger
    of |y_ref| and |y_out|.  The bound alone covers it unless a bias far larger
    than sum_k |xhat_k * what_k| dominates y (a few K-elements): then even the
    correctly rounded bf16 of the exact value can miss it."""
    tol = 8e-3 * bound + 1e-6
    if y_ref is None:
        return tol
    mag = np.maximum(np.abs(y_ref), np.abs(y_out))
    half_ulp = np.ldexp(1.0, (np.floor(np.log2(np.maximum(mag, 2.0 ** -126))) - 8).astype(np.int64))
    return tol + half_ulp


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
