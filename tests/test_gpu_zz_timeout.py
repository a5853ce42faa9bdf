"""Device-side wait limits: with the test hook on, the MMA thread waits on a
barrier that nothing completes ("a flag that nothing sets"); after the wait
limit (1 ms here) the kernel records FG8_ERR_TIMEOUT in the workspace
status word, drains its own copies and tensor-core ops and returns.  The
host reads the status, and the same context then computes correct results
again.  Collected last (file name)."""
import numpy as np
import pytest
import torch

import workloads as W
from conftest import y_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg8():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


def _as_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("entry", ["linear", "fused"])  # fused: the kernels that quantize x in their launch
@pytest.mark.parametrize("M", [16, 640])  # the few-token kernel and the tiled GEMM
@pytest.mark.parametrize("fmt", [0, 1])
def test_wait_limit_reports_timeout_and_context_survives(fg8, orc, M, fmt, entry):
    N, K = 512, 1024
    x = W.x_normal(M, K, seed=M + 1)
    w = W.normal((N, K), 0.02, seed=M + 2)
    wq, ws = fg8.quantize_weight(w.cuda(), fmt)
    if entry == "linear":
        nb = fg8.fg8_linear_workspace_bytes(M, N, K, fmt)
        call = fg8.fg8_linear
    else:
        nb = fg8.fg8_linear_fused_workspace_bytes(M, N, K, fmt)
        call = fg8.fg8_linear_fused
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    xd = x.cuda()
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    try:
        fg8.fg8_set_wait_limit_ns(1_000_000)
        fg8.fg8_set_test_stall(True)
        call(xd.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), 0, y.data_ptr(), N, fmt, wsp.data_ptr(), nb,
             stream=s)
        torch.cuda.synchronize()
        assert fg8.fg8_check_device_status(wsp.data_ptr(), s) == fg8.FG8_ERR_TIMEOUT
    finally:
        fg8.fg8_set_test_stall(False)
        fg8.fg8_set_wait_limit_ns(2_000_000_000)
    # the context is usable and the (re-zeroed) workspace gives correct results
    call(xd.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), 0, y.data_ptr(), N, fmt, wsp.data_ptr(), nb,
         stream=s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsp.data_ptr(), s) == fg8.FG8_OK
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
    y64, bound, _ = orc.linear(W.bf16_bits(x), owq, ows, None, fmt)
    err = np.abs(_as_f64(W.bf16_bits(y.cpu())) - y64)
    assert (err <= y_tolerance(bound)).all()
