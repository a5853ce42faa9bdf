"""Non-default block size (weight_block_size = (32, 32)): 1 x 32 activation
groups and 32 x 32 weight blocks.  Quantizers bit-exact against the oracle
(both scale formats, ragged K and N); the UE8M0 layer against the oracle
on every element over several tiles with ragged edges; float scales
refused for the layer; block 128 through the same calls unchanged."""
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


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _np(t):
    return t.view(torch.uint8).cpu().numpy() if t.element_size() == 1 else t.cpu().numpy()


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(5, 256), (130, 80), (3, 48), (64, 1040)])
def test_act_quant_block32_bits(fg8, orc, fmt, M, K):
    x = W.x_outliers(M, K, seed=M + K).cuda()
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, -(-K // 32), dtype=torch.float32 if fmt == FLOAT else torch.uint8, device="cuda")
    fg8.fg8_quantize_act_block(x.data_ptr(), M, K, K, xq.data_ptr(), xs.data_ptr(), fmt, 32, _stream())
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt, 32)
    assert np.array_equal(xq.cpu().numpy(), oq)
    assert np.array_equal(xs.cpu().numpy(), os_)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("N,K", [(64, 64), (200, 144), (40, 80), (1000, 528)])
def test_weight_quant_block32_bits(fg8, orc, fmt, N, K):
    w = W.w_row_groups(N, K, 0.02, seed=N + 3 * K).cuda()
    wq = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    ws = torch.empty(-(-N // 32), -(-K // 32), dtype=torch.float32 if fmt == FLOAT else torch.uint8, device="cuda")
    fg8.fg8_quantize_weight_block(w.data_ptr(), N, K, K, wq.data_ptr(), ws.data_ptr(), fmt, 32, _stream())
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_weight(W.bf16_bits(w), fmt, 32)
    assert np.array_equal(wq.cpu().numpy(), oq)
    assert np.array_equal(ws.cpu().numpy(), os_)


def _layer(fg8, M, N, K, seed, bias=True, block=32, fmt=UE8M0):
    x = W.x_student_t(M, K, seed=seed).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1).cuda()
    b = W.normal((N,), 0.1, seed=seed + 2).cuda() if bias else None
    wq = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    ws = torch.empty(-(-N // block), -(-K // block), dtype=torch.float32 if fmt == FLOAT else torch.uint8,
                     device="cuda")
    fg8.fg8_quantize_weight_block(w.data_ptr(), N, K, K, wq.data_ptr(), ws.data_ptr(), fmt, block, _stream())
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nb = fg8.fg8_linear_block_workspace_bytes(M, N, K, fmt, block)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    fg8.fg8_linear_block(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), 0 if b is None else b.data_ptr(),
                         y.data_ptr(), N, fmt, block, wsp.data_ptr(), nb, _stream())
    st = fg8.fg8_check_device_status(wsp.data_ptr(), _stream())
    return x, wq, ws, b, y, st


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (300, 264, 400), (129, 520, 1040), (17, 136, 80),
                                   (1000, 1032, 2064)])
def test_linear_block32_vs_oracle(fg8, orc, M, N, K):
    x, wq, ws, b, y, st = _layer(fg8, M, N, K, seed=M + N + K)
    assert st == 0
    y64, bound, _ = orc.linear(W.bf16_bits(x), wq.cpu().numpy(), ws.cpu().numpy(), W.bf16_bits(b), UE8M0, block=32)
    yg = (W.bf16_bits(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(yg - y64)
    bad = ~(err <= y_tolerance(bound))
    assert not bad.any(), f"{bad.sum()} of {bad.size}; worst {np.nanmax(err - y_tolerance(bound))}"


def test_linear_block32_no_bias(fg8, orc):
    x, wq, ws, b, y, st = _layer(fg8, 384, 512, 512, seed=3, bias=False)
    assert st == 0
    y64, bound, _ = orc.linear(W.bf16_bits(x), wq.cpu().numpy(), ws.cpu().numpy(), None, UE8M0, block=32)
    yg = (W.bf16_bits(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert (np.abs(yg - y64) <= y_tolerance(bound)).all()


def test_linear_block32_refuses_float_scales(fg8):
    assert fg8.fg8_linear_block_workspace_bytes(256, 256, 256, FLOAT, 32) == 0
    with pytest.raises(fg8.FG8Error):
        _layer(fg8, 256, 256, 256, seed=5, fmt=FLOAT)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_block128_through_block_calls_is_the_default(fg8, fmt):
    M, N, K = 200, 264, 400
    x, wq, ws, b, y, st = _layer(fg8, M, N, K, seed=9, block=128, fmt=fmt)
    assert st == 0
    y2 = fg8.linear(x, wq.view(torch.float8_e4m3fn), ws if fmt == FLOAT else ws.view(torch.float8_e8m0fnu), b,
                    "ue8m0" if fmt else "float")
    assert torch.equal(y, y2)


def test_layer_wrappers_block32(fg8, orc):
    """quantize_weight / quantize_act / linear / FP8Linear with block = 32."""
    M, N, K = 150, 264, 320
    x = W.x_normal(M, K, seed=11).cuda()
    w = W.normal((N, K), 0.02, seed=12).cuda()
    b = W.normal((N,), 0.1, seed=13).cuda()
    wq, ws = fg8.quantize_weight(w, "ue8m0", block=32)
    assert ws.shape == (-(-N // 32), K // 32)
    oq, os_ = orc.quantize_weight(W.bf16_bits(w), UE8M0, 32)
    assert np.array_equal(_np(wq), oq) and np.array_equal(_np(ws), os_)
    xq, xs = fg8.quantize_act(x, "ue8m0", block=32)
    aq, as_ = orc.quantize_act(W.bf16_bits(x), UE8M0, 32)
    assert np.array_equal(_np(xq), aq) and np.array_equal(_np(xs), as_)
    y = fg8.linear(x, wq, ws, b, "ue8m0", block=32)
    layer = fg8.FP8Linear(w, b, "ue8m0", block=32)
    y2 = layer(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    y64, bound, _ = orc.linear(W.bf16_bits(x), oq, os_, W.bf16_bits(b), UE8M0, block=32)
    yg = (W.bf16_bits(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert (np.abs(yg - y64) <= y_tolerance(bound)).all()
