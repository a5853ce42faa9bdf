"""The few-token path of fg8_linear: the swap-AB split-K kernel that streams
the weights as the tensor core's M side, on the prepare step's quantized
activations (or, for UE8M0 scales and M <= 16, quantizing x itself), for
M <= 32 and up to M = 128 while N is small enough.  Checked against the
oracle on every element, at token counts around each padding step (16, 32,
64, 128), shapes whose K-range is split over many CTAs, ragged weight tiles
and K, and both sides of the shape rule that picks it."""
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


def _bits(t):
    return W.bf16_bits(t.cpu())


def _as_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(orc, x, w, b, y, fmt):
    owq, ows = orc.quantize_weight(_bits(w), fmt)
    y64, bound, _ = orc.linear(_bits(x), owq, ows, None if b is None else _bits(b), fmt)
    err = np.abs(_as_f64(_bits(y)) - y64)
    tol = y_tolerance(bound)
    bad = ~(err <= tol)  # NaN counts as out of tolerance
    assert not bad.any(), f"{bad.sum()} of {bad.size} elements out of tolerance; worst {(err - tol).max()}"


def _run(fg8, orc, M, N, K, fmt, seed, bias=True, gen=W.x_outliers):
    x = gen(M, K, seed=seed).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1).cuda()
    b = W.normal((N,), 0.1, seed=seed + 2).cuda() if bias else None
    wq, ws = fg8.quantize_weight(w, fmt)
    y = fg8.linear(x, wq, ws, b, fmt)
    torch.cuda.synchronize()
    _check(orc, x, w, b, y, fmt)
    return x, w, b, wq, ws, y


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 31, 33, 64, 65, 100, 127, 128])
def test_token_counts(fg8, orc, fmt, M):
    _run(fg8, orc, M, 1040, 1040, fmt, seed=M)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(16, 256, 8192), (5, 384, 2048), (128, 136, 4096), (64, 520, 6160), (1, 8, 16),
                                   (33, 4096, 1024), (3, 1032, 7168), (100, 264, 12288), (1, 256, 16384)])
def test_split_k_shapes(fg8, orc, fmt, M, N, K):
    """Few weight tiles and a long K: the K-range is split over up to 64 CTAs
    (at most 512 / M) whose fp32 partials the last one adds up, with each of
    its three load batchings (M <= 8, M <= 32, larger) and split counts that
    do not fill the last batch; ragged last weight tile, token batch and K."""
    _run(fg8, orc, M, N, K, fmt, seed=N + K)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 2448), (16, 3000, 3200), (32, 9000, 1104), (5, 1032, 16384),
                                   (17, 14336, 4096), (8, 4104, 14336)])
def test_many_tiles_long_k(fg8, orc, fmt, M, N, K):
    """Shapes with at least 4 x 148 (weight tile, K-block) pairs: many weight
    tiles (ragged last tile, K-block and token batch) or few tiles with a
    long K split over up to 16 CTAs.  Repeated calls give the same bits."""
    x, w, b, wq, ws, y = _run(fg8, orc, M, N, K, fmt, seed=M + N + K)
    y2 = fg8.linear(x, wq, ws, b, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_no_bias_and_zero_input(fg8, orc, fmt):
    _run(fg8, orc, 20, 264, 3072, fmt, seed=5, bias=False)
    x = torch.zeros(20, 3072, dtype=torch.bfloat16, device="cuda")
    w = W.normal((264, 3072), 0.02, seed=6).cuda()
    b = W.normal((264,), 0.1, seed=7).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    y = fg8.linear(x, wq, ws, b, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y, b.expand(20, 264))


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_strided_x_and_y(fg8, orc, fmt):
    """x and y with row strides larger than K and N, through the C ABI."""
    M, N, K = 48, 392, 1536
    xf = W.x_student_t(M, K + 64, seed=21).cuda()
    x = xf[:, :K]
    w = W.normal((N, K), 0.02, seed=22).cuda()
    b = W.normal((N,), 0.1, seed=23).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    ld_y = N + 24
    ybuf = torch.full((M, ld_y), float("nan"), dtype=torch.bfloat16, device="cuda")
    nb = fg8.fg8_linear_workspace_bytes(M, N, K, fmt)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    fg8.fg8_linear(x.data_ptr(), M, N, K, x.stride(0), wq.data_ptr(), ws.data_ptr(), b.data_ptr(), ybuf.data_ptr(),
                   ld_y, fmt, wsp.data_ptr(), nb, s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsp.data_ptr(), s) == 0
    assert torch.isnan(ybuf[:, N:].float()).all()  # nothing written past N
    _check(orc, x.contiguous(), w, b, ybuf[:, :N].contiguous(), fmt)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N", [(33, 9472), (33, 9480), (128, 9472), (40, 1040), (20, 1040)])
def test_dispatch_and_prepare_run(fg8, orc, fmt, M, N):
    """Past 32 tokens fg8_linear takes the few-token kernel while the tiled
    GEMM's grid would cover at most a quarter of the SMs (N <= 9472) and the
    tiled GEMM beyond.  Either way fg8_linear_prepare then fg8_linear_run
    (which picks the kernel by the same rule) gives fg8_linear's bits."""
    K = 256
    x, w, b, wq, ws, y = _run(fg8, orc, M, N, K, fmt, seed=M + N)
    nb = fg8.fg8_linear_workspace_bytes(M, N, K, fmt)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    y2 = torch.full_like(y, float("nan"))
    s = torch.cuda.current_stream().cuda_stream
    if fmt == UE8M0 and M <= 16:
        pytest.skip("fg8_linear quantizes inside the few-token kernel here")
    fg8.fg8_linear_prepare(x.data_ptr(), M, N, K, K, ws.data_ptr(), fmt, wsp.data_ptr(), nb, s)  # raises on error
    fg8.fg8_linear_run(wq.data_ptr(), ws.data_ptr(), b.data_ptr(), y2.data_ptr(), M, N, K, N, fmt, wsp.data_ptr(), nb, s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsp.data_ptr(), s) == 0
    assert torch.equal(y, y2)


def test_repeated_calls_same_workspace(fg8, orc):
    """Split-K arrival counters start from zero on every call: back-to-back
    calls on one workspace give identical results."""
    M, N, K = 16, 256, 8192
    x = W.x_normal(M, K, seed=31).cuda()
    w = W.normal((N, K), 0.02, seed=32).cuda()
    wq, ws = fg8.quantize_weight(w, FLOAT)
    nb = fg8.fg8_linear_workspace_bytes(M, N, K, FLOAT)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    ys = [fg8.linear(x, wq, ws, None, FLOAT, workspace=wsp) for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    _check(orc, x, w, None, ys[0], FLOAT)
