"""fg8_linear_noalloc: the layer for callers that cannot allocate device memory.

Such callers (a host framework that owns all device memory in its own pool, or
code that must not call cudaMalloc because it can synchronize the device)
cannot hand fg8_linear a workspace; this entry point uses a fixed scratch
array inside the library instead.  The test calls it through the C ABI several
times in a row, on different shapes, scale formats and kernels (the tiled
GEMM, the few-token split-K kernel and its fused UE8M0 variant), so every
call after the first runs on a scratch that still holds the previous call's
bytes.  Each result is checked against the CPU oracle within the tolerance
every GPU test uses, and against fg8_linear on the same inputs bit for bit
(the same kernels run on the same bytes).  It also checks that a shape beyond
the scratch's 64 MiB and bad arguments are refused with their status.

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
    return (W.bf16_bits(t.cpu()).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _run_and_check(fg8, orc, M, N, K, fmt, seed):
    x = W.x_outliers(M, K, seed=seed)
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1)
    b = W.normal((N,), 0.1, seed=seed + 2)
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    wq, ws = fg8.quantize_weight(wd, fmt)
    stream = torch.cuda.current_stream().cuda_stream
    y_new = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = fg8.lib().fg8_linear_noalloc(xd.data_ptr(), M, N, K, xd.stride(0), wq.data_ptr(), ws.data_ptr(),
                                      bd.data_ptr(), y_new.data_ptr(), y_new.stride(0), fmt, stream)
    assert st == 0, fg8.fg8_status_string(st)
    torch.cuda.synchronize()
    # the oracle: its own weight quantization, the layer in double, the y tolerance
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
    y64, bound, _ = orc.linear(W.bf16_bits(x), owq, ows, W.bf16_bits(b), fmt)
    err = np.abs(_bits_f64(y_new) - y64)
    ok = err <= y_tolerance(bound)
    assert ok.all(), f"M={M} fmt={fmt}: {int((~ok).sum())} elements out of tolerance, max err {np.nanmax(err)}"
    # the existing entry point on the same inputs: the same kernels, so the same bits
    y_ref = fg8.linear(xd, wq, ws, bd, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y_new, y_ref), f"M={M} fmt={fmt}: noalloc differs from fg8_linear"


def test_noalloc_vs_oracle_calls_in_a_row(fg8, orc):
    _run_and_check(fg8, orc, 300, 520, 1040, FLOAT, seed=41)   # tiled GEMM; first call on this device
    _run_and_check(fg8, orc, 129, 256, 480, UE8M0, seed=42)    # tiled GEMM on the scratch the first left
    _run_and_check(fg8, orc, 16, 1040, 2048, FLOAT, seed=43)   # few-token kernel, split-K partials in the scratch
    _run_and_check(fg8, orc, 1, 4096, 1024, FLOAT, seed=44)
    _run_and_check(fg8, orc, 16, 1040, 2048, UE8M0, seed=45)   # fused few-token kernel (quantizes x itself)
    _run_and_check(fg8, orc, 1, 264, 4096, UE8M0, seed=46)
    _run_and_check(fg8, orc, 200, 2048, 4096, FLOAT, seed=48)  # tiled GEMM split over K (partials in the scratch)
    _run_and_check(fg8, orc, 256, 1024, 4096, UE8M0, seed=49)
    _run_and_check(fg8, orc, 300, 520, 1040, FLOAT, seed=47)   # back to the tiled GEMM


def test_noalloc_refuses_shapes_beyond_its_scratch(fg8):
    M, N, K = 8192, 1024, 8192  # needs > 64 MiB of workspace
    assert fg8.fg8_linear_workspace_bytes(M, N, K, FLOAT) > (64 << 20)
    st = fg8.lib().fg8_linear_noalloc(16, M, N, K, K, 16, 16, None, 16, N, FLOAT, None)
    assert st == fg8.FG8_ERR_WORKSPACE


def test_noalloc_checks_arguments_before_anything_else(fg8):
    M, N, K = 64, 256, 256
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    ws = torch.ones((2, 2), dtype=torch.float32, device="cuda")
    L = fg8.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert L.fg8_linear_noalloc(None, M, N, K, K, wq.data_ptr(), ws.data_ptr(), None, y.data_ptr(), N + 8, FLOAT,
                                s) == fg8.FG8_ERR_INVALID_ARG
    assert L.fg8_linear_noalloc(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), None, y.data_ptr() + 2,
                                N + 8, FLOAT, s) == fg8.FG8_ERR_ALIGNMENT
    assert L.fg8_linear_noalloc(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), None, y.data_ptr(), N + 8,
                                7, s) == fg8.FG8_ERR_INVALID_ARG
    assert L.fg8_linear_noalloc(x.data_ptr(), M, N, 200, K, wq.data_ptr(), ws.data_ptr(), None, y.data_ptr(),
                                N + 8, FLOAT, s) == fg8.FG8_ERR_ALIGNMENT
