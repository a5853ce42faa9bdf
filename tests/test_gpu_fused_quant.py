"""fg8_linear_fused: the activation quantization inside the tiled GEMM's
launch.  Checked against the oracle -- the codes and scales the kernel wrote
into the workspace (decoded from the GEMM's layouts) bit for bit, y within
the tolerance -- and against fg8_linear bit for bit, over several calls on
one workspace (the unit flags compare with an epoch that advances per call),
with and without the next layer's requantization, and for the shapes that
run the separate prepare step instead (few tokens, long K)."""
import numpy as np
import pytest
import torch

import workloads as W
from _ws_layout import decode
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


def _s():
    return torch.cuda.current_stream().cuda_stream


def _f64(y):
    return (W.bf16_bits(y.cpu()).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _scale_bits(a, fmt):
    return a.view(np.uint32) if fmt == FLOAT else a


def _same(got, want, what):
    got, want = np.ascontiguousarray(got), np.ascontiguousarray(want)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {tuple(bad[0])}")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(8176, 1920, 480), (300, 520, 1040), (1000, 264, 4096), (129, 4104, 144)])
def test_fused_vs_oracle_and_linear(fg8, orc, fmt, M, N, K):
    w = W.w_row_groups(N, K, 0.02, seed=N + K)
    b = W.normal((N,), 0.1, seed=5)
    wd, bd = w.cuda(), b.cuda()
    wq, ws = fg8.quantize_weight(wd, fmt)
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
    wsp = torch.zeros(fg8.fg8_linear_fused_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")
    for call in range(3):  # one workspace, three calls: the epoch advances each time
        x = W.x_outliers(M, K, seed=17 * call + M)
        xd = x.cuda()
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        fg8.fg8_linear_fused(xd.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), bd.data_ptr(), y.data_ptr(), N,
                             fmt, wsp.data_ptr(), wsp.numel(), stream=_s())
        torch.cuda.synchronize()
        assert fg8.fg8_check_device_status(wsp.data_ptr(), _s()) == 0
        gq, gs = decode(wsp.cpu().numpy(), M, K, fmt)
        oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt)
        _same(gq, oq, f"codes (call {call})")
        _same(gs, _scale_bits(os_, fmt), f"scales (call {call})")
        y64, bound, _ = orc.linear_dequant(oq, os_, owq, ows, W.bf16_bits(b), fmt)
        err = np.abs(_f64(y) - y64)
        assert (err <= y_tolerance(bound)).all(), f"y out of tolerance (call {call}): max err {np.nanmax(err)}"
        assert torch.equal(y, fg8.linear(xd, wq, ws, bd, fmt)), f"call {call}: differs from fg8_linear"


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K1,N1,N2", [(8176, 480, 1920, 480), (300, 256, 528, 136)])
def test_fused_with_next_layer(fg8, orc, fmt, M, K1, N1, N2):
    """x quantized in the first GEMM's launch, y1 requantized in its epilogue:
    both layers equal two fg8_linear calls bit for bit, and y1's codes and
    scales in the next workspace are the oracle's."""
    x = W.x_outliers(M, K1, seed=M + K1).cuda()
    w1 = W.normal((N1, K1), 0.02, seed=N1).cuda()
    w2 = W.w_row_groups(N2, N1, 0.02, seed=N2 + 1).cuda()
    b1 = W.normal((N1,), 0.1, seed=3).cuda()
    b2 = W.normal((N2,), 0.1, seed=4).cuda()
    wq1, ws1 = fg8.quantize_weight(w1, fmt)
    wq2, ws2 = fg8.quantize_weight(w2, fmt)
    wsa = torch.zeros(fg8.fg8_linear_fused_workspace_bytes(M, N1, K1, fmt), dtype=torch.uint8, device="cuda")
    wsb = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N2, N1, fmt), dtype=torch.uint8, device="cuda")
    y1 = torch.empty((M, N1), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, N2), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        fg8.fg8_linear_fused(x.data_ptr(), M, N1, K1, K1, wq1.data_ptr(), ws1.data_ptr(), b1.data_ptr(), y1.data_ptr(),
                             N1, fmt, wsa.data_ptr(), wsa.numel(), N2, ws2.data_ptr(), wsb.data_ptr(), wsb.numel(),
                             _s())
        fg8.fg8_linear_run(wq2.data_ptr(), ws2.data_ptr(), b2.data_ptr(), y2.data_ptr(), M, N2, N1, N2, fmt,
                           wsb.data_ptr(), wsb.numel(), _s())
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsa.data_ptr(), _s()) == 0
    assert fg8.fg8_check_device_status(wsb.data_ptr(), _s()) == 0
    nq, ns = decode(wsb.cpu().numpy(), M, N1, fmt)
    oq, os_ = orc.quantize_act(W.bf16_bits(y1.cpu()), fmt)
    _same(nq, oq, "requantized codes")
    _same(ns, _scale_bits(os_, fmt), "requantized scales")
    r1 = fg8.linear(x, wq1, ws1, b1, fmt)
    r2 = fg8.linear(r1, wq2, ws2, b2, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y1, r1) and torch.equal(y2, r2)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(1, 4104, 1024), (16, 4096, 1040), (9, 264, 4096)])
def test_fused_entry_few_tokens_vs_oracle(fg8, orc, fmt, M, N, K):
    """Up to 16 tokens: the few-token kernel with its own quantizer warps
    (float and UE8M0), every element against the oracle."""
    x = W.x_outliers(M, K, seed=M + K)
    w = W.w_row_groups(N, K, 0.02, seed=N)
    b = W.normal((N,), 0.1, seed=2)
    wq, ws = fg8.quantize_weight(w.cuda(), fmt)
    wsp = torch.zeros(fg8.fg8_linear_fused_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    xd, bd = x.cuda(), b.cuda()
    for _ in range(2):
        fg8.fg8_linear_fused(xd.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), bd.data_ptr(), y.data_ptr(), N,
                             fmt, wsp.data_ptr(), wsp.numel(), stream=_s())
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsp.data_ptr(), _s()) == 0
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
    y64, bound, _ = orc.linear(W.bf16_bits(x), owq, ows, W.bf16_bits(b), fmt)
    err = np.abs(_f64(y) - y64)
    assert (err <= y_tolerance(bound)).all(), f"max err {np.nanmax(err)}"


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(40, 4096, 1024), (1000, 512, 8192)])
def test_fused_entry_on_shapes_that_prepare_separately(fg8, fmt, M, N, K):
    """17 to 128 tokens and long K take fg8_linear's own path through the same entry."""
    x = W.x_normal(M, K, seed=M + K).cuda()
    wq, ws = fg8.quantize_weight(W.normal((N, K), 0.02, seed=N).cuda(), fmt)
    b = W.normal((N,), 0.1, seed=2).cuda()
    wsp = torch.zeros(fg8.fg8_linear_fused_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fg8.fg8_linear_fused(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), b.data_ptr(), y.data_ptr(), N, fmt,
                         wsp.data_ptr(), wsp.numel(), stream=_s())
    torch.cuda.synchronize()
    assert torch.equal(y, fg8.linear(x, wq, ws, b, fmt))
