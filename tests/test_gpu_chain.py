"""Two chained layers (fg8_linear_run_chain): the first layer's GEMM epilogue
quantizes its bf16 output for the second layer.

Checked against the CPU oracle, layer by layer (the ESM-2 "both GEMMs back to
back" reading: the second layer consumes the first layer's bf16 output):
  - y1 against oracle.linear(x), every element, within the y tolerance;
  - the e4m3 codes and scales the epilogue wrote into the second layer's
    workspace against oracle.quantize_act(bits(y1)), bit for bit;
  - y2 against oracle.linear(bits(y1)), every element, within the tolerance.
The chained run must also equal two separate fg8_linear calls bit for bit.
"""
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


def _ws(fg8, M, N, K, fmt):
    return torch.zeros(fg8.fg8_linear_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")


def _f64(y):
    return (W.bf16_bits(y.cpu()).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _scale_bits(a, fmt):
    return a.view(np.uint32) if fmt == FLOAT else a


def _assert_close(y, y64, bound, what):
    got = _f64(y)
    err = np.abs(got - y64)
    tol = y_tolerance(bound)
    bad = ~(err <= tol)
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, first at {np.argwhere(bad)[0]}"


def _assert_same(got, want, what):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: gpu={got[i]!r} oracle={want[i]!r}")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K1,N1,N2", [(8176, 480, 1920, 480), (300, 256, 528, 136), (129, 144, 1040, 264),
                                        (1, 128, 256, 16), (640, 1024, 4096, 1024)])
def test_chain_vs_oracle(fg8, orc, fmt, M, K1, N1, N2):
    x = W.x_outliers(M, K1, seed=M + K1)
    w1 = W.normal((N1, K1), 0.02, seed=N1)
    w2 = W.w_row_groups(N2, N1, 0.02, seed=N2 + 1)
    b1 = W.normal((N1,), 0.1, seed=3)
    b2 = W.normal((N2,), 0.1, seed=4)
    xd, w1d, w2d, b1d, b2d = (t.cuda() for t in (x, w1, w2, b1, b2))
    wq1, ws1 = fg8.quantize_weight(w1d, fmt)
    wq2, ws2 = fg8.quantize_weight(w2d, fmt)
    s = torch.cuda.current_stream().cuda_stream
    wsa, wsb = _ws(fg8, M, N1, K1, fmt), _ws(fg8, M, N2, N1, fmt)
    wsb.fill_(0xFF)  # stale bytes everywhere: the chain must write all it uses
    wsb[:1024].zero_()
    y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
    y2 = torch.full((M, N2), float("nan"), dtype=torch.bfloat16, device="cuda")
    fg8.fg8_linear_prepare(xd.data_ptr(), M, N1, K1, xd.stride(0), ws1.data_ptr(), fmt, wsa.data_ptr(), wsa.numel(), s)
    fg8.fg8_linear_run_chain(wq1.data_ptr(), ws1.data_ptr(), b1d.data_ptr(), y1.data_ptr(), M, N1, K1, N1, fmt,
                             wsa.data_ptr(), wsa.numel(), N2, ws2.data_ptr(), wsb.data_ptr(), wsb.numel(), s)
    torch.cuda.synchronize()
    nxq, nxs = decode(wsb.cpu().numpy(), M, N1, fmt)  # what the epilogue wrote for layer 2
    fg8.fg8_linear_run(wq2.data_ptr(), ws2.data_ptr(), b2d.data_ptr(), y2.data_ptr(), M, N2, N1, N2, fmt,
                       wsb.data_ptr(), wsb.numel(), s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsa.data_ptr(), s) == 0
    assert fg8.fg8_check_device_status(wsb.data_ptr(), s) == 0

    # the oracle, layer by layer (weights quantized by the oracle itself)
    owq1, ows1 = orc.quantize_weight(W.bf16_bits(w1), fmt)
    owq2, ows2 = orc.quantize_weight(W.bf16_bits(w2), fmt)
    y1_64, bound1, _ = orc.linear(W.bf16_bits(x), owq1, ows1, W.bf16_bits(b1), fmt)
    _assert_close(y1, y1_64, bound1, "y1")
    y1_bits = W.bf16_bits(y1.cpu())
    oxq, oxs = orc.quantize_act(y1_bits, fmt)
    _assert_same(np.ascontiguousarray(nxq), oxq, "requantized codes of y1")
    _assert_same(np.ascontiguousarray(nxs), _scale_bits(oxs, fmt), "requantized scales of y1")
    y2_64, bound2, _ = orc.linear_dequant(oxq, oxs, owq2, ows2, W.bf16_bits(b2), fmt)
    _assert_close(y2, y2_64, bound2, "y2")

    # and the chain is the two separate layers, bit for bit
    y1_ref = fg8.linear(xd, wq1, ws1, b1d, fmt)
    y2_ref = fg8.linear(y1_ref, wq2, ws2, b2d, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y1, y1_ref)
    assert torch.equal(y2, y2_ref)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_linear_chain_three_layers_vs_oracle(fg8, orc, fmt):
    """linear_chain over three layers (one without bias): each layer's output
    against the oracle on the previous layer's bf16 output, and equal to
    separate fg8.linear calls."""
    M, dims = 777, [384, 1024, 272, 512]
    x = W.x_student_t(M, dims[0], seed=11)
    layers, host = [], []
    for i in range(3):
        w = W.w_row_groups(dims[i + 1], dims[i], 0.03, seed=20 + i)
        b = None if i == 1 else W.normal((dims[i + 1],), 0.1, seed=30 + i)
        wq, ws = fg8.quantize_weight(w.cuda(), fmt)
        layers.append((wq, ws, None if b is None else b.cuda()))
        host.append((w, b))
    ys = fg8.linear_chain(x.cuda(), layers, fmt)
    torch.cuda.synchronize()
    a = W.bf16_bits(x)
    ref = x.cuda()
    for (wq, ws, bd), (w, b), y in zip(layers, host, ys):
        owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
        y64, bound, _ = orc.linear(a, owq, ows, None if b is None else W.bf16_bits(b), fmt)
        _assert_close(y, y64, bound, "layer output")
        a = W.bf16_bits(y.cpu())
        ref = fg8.linear(ref, wq, ws, bd, fmt)
        assert torch.equal(y, ref)
