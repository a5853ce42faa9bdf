"""Checkpoint conversions on the GPU against the oracle, bit for bit:
Fp8Dequantize (block scales folded into bf16 weights) and the float32 ->
UE8M0 scale conversion ([zh] §五, §七)."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

FLOAT, UE8M0 = 0, 1


@pytest.fixture(scope="module")
def fg8():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("N,K", [(1, 16), (200, 144), (256, 384), (1920, 480), (4099, 1040)])
def test_dequantize_matches_oracle(fg8, orc, fmt, N, K):
    w = W.w_row_groups(N, K, 0.02, seed=N + K)
    wq, ws = orc.quantize_weight(W.bf16_bits(w), fmt)
    want = orc.dequantize_weight(wq, ws, fmt)
    wq_t = torch.from_numpy(wq).cuda()
    ws_t = torch.from_numpy(np.ascontiguousarray(ws)).cuda()
    if fmt == UE8M0:
        ws_t = ws_t.view(torch.float8_e8m0fnu)
    got = fg8.dequantize_weight(wq_t.view(torch.float8_e4m3fn), ws_t, fmt)
    torch.cuda.synchronize()
    assert np.array_equal(W.bf16_bits(got.cpu()), want)


def test_dequantize_of_device_quantized_weight_with_row_stride(fg8, orc):
    """The device quantizer's output dequantized into a wider buffer."""
    N, K = 300, 256
    w = W.normal((N, K), 0.05, seed=5).cuda()
    wq, ws = fg8.quantize_weight(w, FLOAT)
    out = torch.full((N, K + 40), float("nan"), dtype=torch.bfloat16, device="cuda")
    fg8.fg8_dequantize_weight(wq.data_ptr(), N, K, ws.data_ptr(), FLOAT, out.data_ptr(), K + 40,
                              torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    want = orc.dequantize_weight(wq.cpu().view(torch.uint8).numpy(), ws.cpu().numpy(), FLOAT)
    assert np.array_equal(W.bf16_bits(out[:, :K].contiguous().cpu()), want)
    assert torch.isnan(out[:, K:].float()).all()


def test_scale_to_ue8m0_matches_oracle(fg8, orc):
    g = np.random.default_rng(7)
    e = g.integers(-127, 128, size=5000)
    s = np.ldexp(np.float32(1.0), e).astype(np.float32)
    bad_idx = g.choice(s.size, size=300, replace=False)
    junk = np.array([3.0, 0.0, -1.0, np.inf, np.nan, 2.0 ** -128, 1.5, -0.0], dtype=np.float32)
    s[bad_idx] = junk[np.arange(bad_idx.size) % junk.size]
    want, want_bad = orc.scale_to_e8m0(s)
    got, got_bad = fg8.scale_to_ue8m0(torch.from_numpy(s).cuda())
    assert np.array_equal(got.view(torch.uint8).cpu().numpy(), want)
    assert got_bad == want_bad == 300
