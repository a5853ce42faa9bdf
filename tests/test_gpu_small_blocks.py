"""Non-default block sizes (weight_block_size = (32, 32) and (64, 64)): 1 x b
activation groups and b x b weight blocks, float32 or UE8M0 scales.

Quantizers bit-exact against the oracle (both scale formats, ragged K and N,
enough groups for several passes of the grid); the layer against the oracle
on every element over several tiles with ragged edges, with float scales
promoted per b-wide slice of K and UE8M0 scales applied by the block-scaled
MMA; block 128 through the same calls unchanged."""
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


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(5, 256), (130, 80), (3, 48), (64, 1040), (3000, 4112)])
def test_act_quant_small_block_bits(fg8, orc, fmt, M, K, blk):
    x = W.x_outliers(M, K, seed=M + K + blk).cuda()
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, -(-K // blk), dtype=torch.float32 if fmt == FLOAT else torch.uint8, device="cuda")
    fg8.fg8_quantize_act_block(x.data_ptr(), M, K, K, xq.data_ptr(), xs.data_ptr(), fmt, blk, _stream())
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt, blk)
    assert np.array_equal(xq.cpu().numpy(), oq)
    assert np.array_equal(_np(xs).view(np.uint32) if fmt == FLOAT else _np(xs),
                          os_.view(np.uint32) if fmt == FLOAT else os_)


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("N,K", [(64, 64), (200, 144), (40, 80), (1000, 528), (136, 208)])
def test_weight_quant_small_block_bits(fg8, orc, fmt, N, K, blk):
    w = W.w_row_groups(N, K, 0.02, seed=N + 3 * K + blk).cuda()
    wq = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    ws = torch.empty(-(-N // blk), -(-K // blk), dtype=torch.float32 if fmt == FLOAT else torch.uint8, device="cuda")
    fg8.fg8_quantize_weight_block(w.data_ptr(), N, K, K, wq.data_ptr(), ws.data_ptr(), fmt, blk, _stream())
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_weight(W.bf16_bits(w), fmt, blk)
    assert np.array_equal(wq.cpu().numpy(), oq)
    assert np.array_equal(_np(ws).view(np.uint32) if fmt == FLOAT else _np(ws),
                          os_.view(np.uint32) if fmt == FLOAT else os_)


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


def _check_vs_oracle(orc, x, wq, ws, b, y, fmt, block):
    y64, bound, _ = orc.linear(W.bf16_bits(x), wq.cpu().numpy(), _np(ws), None if b is None else W.bf16_bits(b),
                               fmt, block=block)
    yg = (W.bf16_bits(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(yg - y64)
    bad = ~(err <= y_tolerance(bound))
    assert not bad.any(), f"{bad.sum()} of {bad.size}; worst {np.nanmax(err - y_tolerance(bound))}"


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K,bias", [(256, 256, 256, True), (300, 264, 400, True), (129, 520, 1040, True),
                                        (17, 136, 80, True), (1000, 1032, 2064, True), (520, 4104, 48, False)])
def test_linear_small_block_vs_oracle(fg8, orc, fmt, M, N, K, bias, blk):
    """Every element; float scales differ per blk-slice of K and per blk-block of
    N, so a slice promoted with the wrong scale fails.  (The 48-channel case,
    one and a half 32-slices, runs without bias: with so few terms a bias-
    dominated output's bf16 rounding alone can exceed 8e-3 * sum|xhat*what|,
    the acceptance rule's edge case.)"""
    x, wq, ws, b, y, st = _layer(fg8, M, N, K, seed=M + N + K + blk, block=blk, fmt=fmt, bias=bias)
    assert st == 0
    _check_vs_oracle(orc, x, wq, ws, b, y, fmt, blk)


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_linear_small_block_no_bias(fg8, orc, fmt, blk):
    x, wq, ws, b, y, st = _layer(fg8, 384, 512, 512, seed=3, bias=False, block=blk, fmt=fmt)
    assert st == 0
    _check_vs_oracle(orc, x, wq, ws, None, y, fmt, blk)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_block128_through_block_calls_is_the_default(fg8, fmt):
    M, N, K = 200, 264, 400
    x, wq, ws, b, y, st = _layer(fg8, M, N, K, seed=9, block=128, fmt=fmt)
    assert st == 0
    y2 = fg8.linear(x, wq.view(torch.float8_e4m3fn), ws if fmt == FLOAT else ws.view(torch.float8_e8m0fnu), b,
                    "ue8m0" if fmt else "float")
    assert torch.equal(y, y2)


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("sfmt", ["float", "ue8m0"])
def test_layer_wrappers_small_blocks(fg8, orc, sfmt, blk):
    """quantize_weight / quantize_act / linear / FP8Linear at block 32 and 64."""
    fmt = 1 if sfmt == "ue8m0" else 0
    M, N, K = 150, 264, 320
    x = W.x_normal(M, K, seed=11).cuda()
    w = W.normal((N, K), 0.02, seed=12).cuda()
    b = W.normal((N,), 0.1, seed=13).cuda()
    wq, ws = fg8.quantize_weight(w, sfmt, block=blk)
    assert ws.shape == (-(-N // blk), K // blk)
    oq, os_ = orc.quantize_weight(W.bf16_bits(w), fmt, blk)
    assert np.array_equal(_np(wq), oq) and np.array_equal(_np(ws), os_)
    xq, xs = fg8.quantize_act(x, sfmt, block=blk)
    aq, as_ = orc.quantize_act(W.bf16_bits(x), fmt, blk)
    assert np.array_equal(_np(xq), aq) and np.array_equal(_np(xs), as_)
    y = fg8.linear(x, wq, ws, b, sfmt, block=blk)
    layer = fg8.FP8Linear(w, b, sfmt, block=blk)
    y2 = layer(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    y64, bound, _ = orc.linear(W.bf16_bits(x), oq, os_, W.bf16_bits(b), fmt, block=blk)
    yg = (W.bf16_bits(y).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert (np.abs(yg - y64) <= y_tolerance(bound)).all()
