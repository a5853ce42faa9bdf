"""Static activation scheme on the GPU ([zh] §四 activation_scheme "static"):
one precomputed scale for the whole tensor.  Bytes bit-exact against the
oracle (saturating values included); the linear layer within the y
tolerance of the oracle's dequantized GEMM."""
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


@pytest.mark.parametrize("M,K,scale", [(1, 16, 0.01), (77, 480, 0.0173), (300, 1040, 0.5), (8, 4096, 2.0 ** -5)])
def test_quantize_act_static_bytes(fg8, orc, M, K, scale):
    x = W.x_outliers(M, K, seed=M + K)  # 20x outlier channels: some values saturate at small scales
    s = torch.tensor([scale], dtype=torch.float32, device="cuda")
    xq, xs = fg8.quantize_act_static(x.cuda(), s)
    torch.cuda.synchronize()
    oq, oxs = orc.quantize_act_static(W.bf16_bits(x), scale)
    assert np.array_equal(xq.view(torch.uint8).cpu().numpy(), oq)
    assert np.array_equal(xs.cpu().numpy(), oxs)


@pytest.mark.parametrize("M,N,K", [(16, 256, 256), (300, 520, 1040), (8176, 1920, 480)])
def test_linear_static_vs_oracle(fg8, orc, M, N, K):
    x = W.x_normal(M, K, seed=3 * M + K)
    w = W.w_row_groups(N, K, 0.02, seed=N + K)
    b = W.normal((N,), 0.1, seed=N)
    scale = float(np.float32(4.0 / 448.0))  # |x| up to ~4 maps onto the e4m3 range; the tail saturates
    s = torch.tensor([scale], dtype=torch.float32, device="cuda")
    wq, ws = fg8.quantize_weight(w.cuda(), "float")
    y = fg8.linear_static(x.cuda(), s, wq, ws, b.cuda())
    torch.cuda.synchronize()
    oq, oxs = orc.quantize_act_static(W.bf16_bits(x), scale)
    rows = np.arange(M) if M <= 512 else np.unique(np.r_[np.arange(0, M, 97), [M - 1, 127, 128]])
    y64, bound, _ = orc.linear_dequant(oq, oxs, wq.view(torch.uint8).cpu().numpy(), ws.cpu().numpy(),
                                       W.bf16_bits(b), 0, rows=rows)
    err = np.abs(_as_f64(W.bf16_bits(y.cpu())[rows]) - y64)
    assert (err <= y_tolerance(bound)).all()
