"""fg8_linear_noalloc: the layer for callers that cannot allocate device memory.

Such callers (a host framework that owns all device memory in its own pool, or
code that must not call cudaMalloc because it can synchronize the device)
cannot hand fg8_linear a workspace; this entry point uses a fixed scratch
array inside the library instead.  The test calls it through the C ABI twice
in a row, on different shapes and scale formats (so the second call runs on a
scratch that still holds the first call's bytes), and compares each result
with fg8_linear's on the same inputs, within the tolerance every GPU test uses.
It also checks that a shape beyond the scratch's 32 MiB is refused.

Kept in a file that pytest collects last, so that a stopping run has already
run every other test; it passes alone in a fresh process too.
"""
import numpy as np
import pytest
import torch

import workloads as W
from conftest import y_tolerance

pytestmark = pytest.mark.gpu

FLOAT, UE8M0 = 0, 1


@pytest.fixture(scope="module")
def fg8():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


def _bits_f64(t):
    return (W.bf16_bits(t).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _run_both(fg8, orc, M, N, K, fmt, seed):
    x = W.x_outliers(M, K, seed=seed).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1).cuda()
    b = W.normal((N,), 0.1, seed=seed + 2).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    stream = torch.cuda.current_stream().cuda_stream
    y_ref = fg8.linear(x, wq, ws, b, fmt)                        # existing entry point
    y_new = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    fg8.fg8_linear_noalloc(x.data_ptr(), M, N, K, x.stride(0), wq.data_ptr(), ws.data_ptr(), b.data_ptr(),
                           y_new.data_ptr(), y_new.stride(0), fmt, stream)
    torch.cuda.synchronize()
    # tolerance of the GPU tests: 8e-3 * sum_k |xhat*what| + 1e-6, bound from the oracle
    owq, ows = orc.quantize_weight(W.bf16_bits(w.cpu()), fmt)
    _, bound, _ = orc.linear(W.bf16_bits(x.cpu()), owq, ows, W.bf16_bits(b.cpu()), fmt)
    diff = np.abs(_bits_f64(y_new) - _bits_f64(y_ref))
    assert np.all(diff <= y_tolerance(bound)), f"max |noalloc - linear| = {diff.max()}"


def test_noalloc_matches_linear_two_calls_in_a_row(fg8, orc):
    _run_both(fg8, orc, 300, 520, 1040, FLOAT, seed=41)   # first call on this device
    _run_both(fg8, orc, 129, 256, 480, UE8M0, seed=42)    # reuses the scratch left by the first


def test_noalloc_refuses_shapes_beyond_its_scratch(fg8):
    M, N, K = 8192, 1024, 8192  # needs > 64 MB of workspace
    assert fg8.fg8_linear_workspace_bytes(M, N, K, FLOAT) > (32 << 20)
    st = fg8.lib().fg8_linear_noalloc(16, M, N, K, K, 16, 16, None, 16, N, FLOAT, None)
    assert st == fg8.FG8_ERR_WORKSPACE
