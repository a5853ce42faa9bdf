"""GPU quantizers vs the CPU oracle: e4m3 bytes and scales must match bit for bit.

Scales are compared as bit patterns (float32 words or UE8M0 bytes), codes as
bytes, over ragged shapes, the pages' model shapes, and every finite bf16 bit
pattern (so every rounding case of the cast is exercised).
"""
import numpy as np
import pytest
import torch

import workloads as W
from _ws_layout import decode

pytestmark = pytest.mark.gpu

FLOAT, UE8M0 = 0, 1


@pytest.fixture(scope="module")
def fg8():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


def _u8(t):
    return t.view(torch.uint8).cpu().numpy()


def _scale_bits(t, fmt):
    a = t.cpu()
    if fmt == FLOAT:
        return a.numpy().view(np.uint32)
    return a.view(torch.uint8).numpy()


def _oracle_scale_bits(a, fmt):
    return a.view(np.uint32) if fmt == FLOAT else a


def _assert_same(got, want, what):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: gpu={got[i]!r} oracle={want[i]!r}")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(16, 256), (1, 16), (129, 144), (3, 1920), (64, 7168), (8176, 480), (257, 1040)])
def test_act_quant_bitexact(fg8, orc, fmt, M, K):
    x = W.x_outliers(M, K, seed=M + K)
    xq, xs = fg8.quantize_act(x.cuda(), fmt)
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt)
    _assert_same(_u8(xq), oq, "xq")
    _assert_same(_scale_bits(xs, fmt), _oracle_scale_bits(os_, fmt), "x_scale")


# The launcher caps the grid at 8 CTAs per SM (64 groups of 128 per CTA, so
# 75,776 groups per pass over 148 SMs; 256 groups of 32 per CTA, 303,104 per
# pass): these shapes need 6 and more passes of the grid-stride loop.
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(8192, 7168), (4096, 14336), (24000, 1040)])
def test_act_quant_bitexact_multi_pass(fg8, orc, fmt, M, K):
    x = W.x_student_t(M, K, seed=M + K)
    assert M * ((K + 127) // 128) > 2 * 75776
    xq, xs = fg8.quantize_act(x.cuda(), fmt)
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt)
    _assert_same(_u8(xq), oq, "xq")
    _assert_same(_scale_bits(xs, fmt), _oracle_scale_bits(os_, fmt), "x_scale")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_act_quant_block32_multi_pass(fg8, orc, fmt):
    M, K = 4096, 4112  # 4096 x 129 groups of 32 = 528,384 groups; ragged last group
    x = W.x_outliers(M, K, seed=77)
    xq, xs = fg8.quantize_act(x.cuda(), fmt, block=32)
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt, block=32)
    _assert_same(_u8(xq), oq, "xq")
    _assert_same(_scale_bits(xs, fmt), _oracle_scale_bits(os_, fmt), "x_scale")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(8192, 7168), (300, 1040)])
def test_prepare_layouts_vs_oracle(fg8, orc, fmt, M, K):
    """The prepare step of fg8_linear writes the codes and, in the GEMM's own
    layouts (K-major float32, or UE8M0 scale-factor tiles), the scales: decoded
    back to row-major they must be the oracle's bit for bit, across every pass
    of the grid."""
    N = 256
    x = W.x_outliers(M, K, seed=M + 2 * K)
    ws_scale = torch.ones(((N + 127) // 128, (K + 127) // 128), dtype=torch.float32, device="cuda")
    if fmt == UE8M0:
        ws_scale = torch.full(ws_scale.shape, 127, dtype=torch.uint8, device="cuda")
    wsp = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    fg8.fg8_linear_prepare(xd.data_ptr(), M, N, K, xd.stride(0), ws_scale.data_ptr(), fmt, wsp.data_ptr(),
                           wsp.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    gq, gs = decode(wsp.cpu().numpy(), M, K, fmt)
    oq, os_ = orc.quantize_act(W.bf16_bits(x), fmt)
    _assert_same(np.ascontiguousarray(gq), oq, "xq in the workspace")
    _assert_same(np.ascontiguousarray(gs), _oracle_scale_bits(os_, fmt), "x scales in the workspace")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_act_quant_every_bf16_pattern(fg8, orc, fmt):
    """All finite bf16 values, shuffled into 128-wide groups, plus groups of
    zeros, signed zeros and subnormals."""
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    finite = bits[np.isfinite(f)].astype(np.uint16)
    rng = np.random.default_rng(5)
    rng.shuffle(finite)
    n = (finite.size + 127) // 128 * 128
    pad = np.zeros(n - finite.size, dtype=np.uint16)
    rows = np.concatenate([finite, pad]).reshape(-1, 128)
    special = np.zeros((4, 128), dtype=np.uint16)
    special[1, ::2] = 0x8000                     # -0.0
    special[2, :] = np.arange(1, 129)            # subnormals
    special[3, :] = 0x8000 | np.arange(1, 129)   # negative subnormals
    # magnitude-limited groups: only small values, so the scale is small too
    small = finite[(finite & 0x7F80) < 0x3000][: 128 * 64].reshape(-1, 128)
    xb = np.concatenate([rows, special, small]).reshape(-1, 256)
    x = W.from_bits(xb).cuda()
    xq, xs = fg8.quantize_act(x, fmt)
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(xb, fmt)
    _assert_same(_u8(xq), oq, "xq")
    _assert_same(_scale_bits(xs, fmt), _oracle_scale_bits(os_, fmt), "x_scale")


def test_act_quant_strided_input(fg8, orc):
    x_full = W.x_normal(40, 512, seed=3)
    x = x_full[:, 64:64 + 384]           # ld_x = 512, 16-byte aligned start
    xq, xs = fg8.quantize_act(x_full.cuda()[:, 64:64 + 384], FLOAT)
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_act(W.bf16_bits(x.contiguous()), FLOAT)
    _assert_same(_u8(xq), oq, "xq")
    _assert_same(_scale_bits(xs, FLOAT), _oracle_scale_bits(os_, FLOAT), "x_scale")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("N,K", [(256, 256), (1920, 480), (480, 1920), (200, 144), (136, 16), (4096, 128)])
def test_weight_quant_bitexact(fg8, orc, fmt, N, K):
    w = W.w_row_groups(N, K, 0.015, seed=N + 3 * K)
    wq, ws = fg8.quantize_weight(w.cuda(), fmt)
    torch.cuda.synchronize()
    oq, os_ = orc.quantize_weight(W.bf16_bits(w), fmt)
    _assert_same(_u8(wq), oq, "wq")
    _assert_same(_scale_bits(ws, fmt), _oracle_scale_bits(os_, fmt), "w_scale_inv")
