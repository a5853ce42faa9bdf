"""GPU linear layer vs the CPU oracle.

Every checked element must satisfy |y_gpu - y_ref| <= 8e-3 * sum_k |xhat_k what_k| + 1e-6,
with y_ref the oracle's double-precision result on its own quantization of
the same bf16 inputs.  Small shapes are checked in full (several tiles,
ragged M/N/K tails); the full-size configurations are checked on sampled
rows (tile boundaries included) in the same launch configuration the bench
times, with the quantized weights compared byte for byte in full.
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


def _bits(t):
    return W.bf16_bits(t)


def _as_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_y(y_gpu_bits, y64, bound, what=""):
    got = _as_f64(y_gpu_bits)
    err = np.abs(got - y64)
    tol = y_tolerance(bound)
    bad = ~(err <= tol)  # NaN counts as out of tolerance
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; first {i}: "
                             f"gpu={got[i]} ref={y64[i]} bound={bound[i]} err={err[i]}")
    return float((err / np.maximum(bound, 1e-30)).max())


def run_case(fg8, orc, x, w, bias, fmt, rows=None):
    """Quantize W and run the layer on the GPU; oracle on the same bf16 inputs."""
    xd, wd = x.cuda(), w.cuda()
    bd = None if bias is None else bias.cuda()
    wq, ws = fg8.quantize_weight(wd, fmt)
    y = fg8.linear(xd, wq, ws, bd, fmt)
    torch.cuda.synchronize()
    owq, ows = orc.quantize_weight(_bits(w), fmt)
    assert np.array_equal(wq.view(torch.uint8).cpu().numpy(), owq)
    y64, bound, _ = orc.linear(_bits(x), owq, ows, None if bias is None else _bits(bias), fmt, rows=rows)
    yb = _bits(y)
    if rows is not None:
        yb = yb[rows]
    return check_y(yb, y64, bound), y


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_tiny_config(fg8, orc, fmt):
    g = W.TINY
    x, w, b = W.make_inputs("tiny", g)
    run_case(fg8, orc, x, w, b, fmt)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (129, 136, 144), (300, 520, 1040), (256, 384, 480), (77, 1920, 480),
                                   (200, 480, 1920), (1, 4096, 384), (640, 264, 256)])
def test_ragged_shapes(fg8, orc, fmt, M, N, K):
    x = W.x_outliers(M, K, seed=M * 7 + K)
    w = W.w_row_groups(N, K, 0.02, seed=N + K)
    b = W.normal((N,), 0.1, seed=N)
    run_case(fg8, orc, x, w, b, fmt)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_no_bias(fg8, orc, fmt):
    x = W.x_normal(130, 256, seed=1)
    w = W.normal((256, 256), 0.02, seed=2)
    run_case(fg8, orc, x, w, None, fmt)


def test_zero_input_gives_bias(fg8):
    x = torch.zeros(130, 256, dtype=torch.bfloat16, device="cuda")
    w = W.normal((264, 256), 0.02, seed=2).cuda()
    b = W.normal((264,), 0.1, seed=3).cuda()
    for fmt in (FLOAT, UE8M0):
        wq, ws = fg8.quantize_weight(w, fmt)
        y = fg8.linear(x, wq, ws, b, fmt)
        assert torch.equal(y, b.expand(130, 264))


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_prequant_gemm_equals_linear(fg8, fmt):
    """fg8_gemm_prequant on fg8_quantize_act's output gives fg8_linear's y, bit for bit."""
    x = W.x_outliers(300, 1040, seed=9).cuda()
    w = W.normal((520, 1040), 0.02, seed=10).cuda()
    b = W.normal((520,), 0.1, seed=11).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    y1 = fg8.linear(x, wq, ws, b, fmt)
    xq, xs = fg8.quantize_act(x, fmt)
    y2 = fg8.gemm_prequant(xq, xs, wq, ws, b, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_float_scales_not_rounded_to_pow2(fg8, orc):
    """Float scales must be applied as given, not rounded up to UE8M0 without
    requantizing ([zh] §七 补充): the GPU result matches the oracle and is far
    from what the rounded scales would give."""
    M, N, K = 128, 256, 512
    x = W.x_normal(M, K, seed=4)
    w = W.normal((N, K), 0.02, seed=5)
    _, y = run_case(fg8, orc, x, w, None, FLOAT)
    oq, os_ = orc.quantize_act(_bits(x), FLOAT)
    owq, ows = orc.quantize_weight(_bits(w), FLOAT)
    up = lambda s: np.array([orc.e8m0_value(orc.e8m0_ceil_byte(v)) for v in s.ravel()], np.float32).reshape(s.shape)
    y_wrong, bound, _ = orc.linear_dequant(oq, up(os_), owq, up(ows), None, FLOAT)
    err = np.abs(_as_f64(_bits(y)) - y_wrong)
    assert (err > y_tolerance(bound)).mean() > 0.5


def test_multiple_calls_and_streams(fg8, orc):
    x = W.x_normal(256, 256, seed=12)
    w = W.normal((256, 256), 0.02, seed=13)
    wq, ws = fg8.quantize_weight(w.cuda(), FLOAT)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ys = [fg8.linear(x.cuda(), wq, ws, None, FLOAT) for _ in range(3)]
    s.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


# ------------------------------------------------------- full-size, sampled --
def _sample_rows(M, n=12, seed=0):
    base = {0, min(127, M - 1), min(128, M - 1), M - 1, M // 2}
    rng = np.random.default_rng(seed)
    extra = rng.integers(0, M, size=n)
    return np.array(sorted(base | set(int(v) for v in extra)), dtype=np.int64)


def full_size_case(fg8, orc, cfg, gemm, stage=1):
    x, w, b = W.make_inputs(cfg, gemm, device="cuda", stage=stage)
    fmt = gemm.fmt
    wq, ws = fg8.quantize_weight(w, fmt)
    y = fg8.linear(x, wq, ws, b, fmt)
    torch.cuda.synchronize()
    wb = _bits(w)
    owq, ows = orc.quantize_weight(wb, fmt)
    assert np.array_equal(wq.view(torch.uint8).cpu().numpy(), owq), "wq differs"
    rows = _sample_rows(gemm.M)
    xb = _bits(x)
    y64, bound, _ = orc.linear(xb, owq, ows, _bits(b), fmt, rows=rows)
    return check_y(_bits(y)[rows], y64, bound, gemm.name)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(8192, 2176, 256), (8192, 384, 1040), (8192, 480, 384)])
def test_wide_tiles_ragged_n(fg8, orc, fmt, M, N, K):
    """Shapes whose tile choice is 256 columns wide with a ragged last tile
    (half or fully past N), sampled rows."""
    x = W.x_outliers(M, K, seed=M + N + K).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=N * 3 + K).cuda()
    b = W.normal((N,), 0.1, seed=N + 1).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    y = fg8.linear(x, wq, ws, b, fmt)
    torch.cuda.synchronize()
    owq, ows = orc.quantize_weight(_bits(w), fmt)
    rows = _sample_rows(M, n=24, seed=N)
    y64, bound, _ = orc.linear(_bits(x), owq, ows, _bits(b), fmt, rows=rows)
    check_y(_bits(y)[rows], y64, bound, f"{M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(2176, 2304, 384), (4000, 2560, 1040), (8176, 1920, 480)])
def test_ragged_row_tiles(fg8, orc, M, N, K):
    """Float shapes whose last 128-row tile is partly past M (and whose last
    256 rows straddle M), ragged K, the ESM-2 shape; sampled rows around the
    tile boundaries."""
    x = W.x_outliers(M, K, seed=M + 2 * K).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=N + 5 * K).cuda()
    b = W.normal((N,), 0.1, seed=N + 7).cuda()
    wq, ws = fg8.quantize_weight(w, FLOAT)
    y = fg8.linear(x, wq, ws, b, FLOAT)
    torch.cuda.synchronize()
    owq, ows = orc.quantize_weight(_bits(w), FLOAT)
    rows = np.unique(np.concatenate([_sample_rows(M, n=24, seed=K), [M - 129, M - 128, M - 1, 255, 256]]))
    rows = rows[(rows >= 0) & (rows < M)].astype(np.int64)
    y64, bound, _ = orc.linear(_bits(x), owq, ows, _bits(b), FLOAT, rows=rows)
    check_y(_bits(y)[rows], y64, bound, f"{M}x{N}x{K}")


@pytest.mark.parametrize("stage", [1, 2])
def test_fullsize_esm2(fg8, orc, stage):
    g = W.ESM_W1 if stage == 1 else W.ESM_W2
    full_size_case(fg8, orc, "esm2", g, stage)


@pytest.mark.parametrize("M", W.LLAMA_M)
@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_fullsize_llama(fg8, orc, M, which):
    full_size_case(fg8, orc, "llama", W.llama(M, which), 1 if which == "gate_up" else 2)


@pytest.mark.parametrize("stage", [1, 2])
def test_fullsize_dsv3(fg8, orc, stage):
    full_size_case(fg8, orc, "dsv3", W.DSV3_UP if stage == 1 else W.DSV3_DOWN, stage)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M", W.SQUARE_M)
def test_fullsize_square(fg8, orc, M, fmt):
    full_size_case(fg8, orc, "square", W.square(M, fmt), 1)



def _dequant(q, s, block=128):
    """value(q) * scale, the scales expanded over their groups/blocks (fp32, on the GPU)."""
    v = q.float()
    sc = s.float()
    rows = sc.repeat_interleave(block, dim=0)[:v.shape[0]] if sc.shape[0] != v.shape[0] else sc
    return v * rows.repeat_interleave(block, dim=1)[:, :v.shape[1]]


@pytest.mark.parametrize("cfg,gemm,stage", [("square", W.square(8192, FLOAT), 1), ("square", W.square(8192, UE8M0), 1),
                                            ("dsv3", W.DSV3_UP, 1), ("llama", W.llama(4096, "gate_up"), 1),
                                            ("esm2", W.ESM_W2, 2)])
def test_fullsize_every_element_vs_fp32_matmul(fg8, cfg, gemm, stage):
    """A library check beside the oracle's sampled rows: every element of y at
    full size against an fp32 matmul (TF32 off) of the dequantized operands,
    y_ref = x^ . w^T + bias, with the same tolerance 8e-3 * (|x^| . |w^|^T) + 1e-6."""
    x, w, b = W.make_inputs(cfg, gemm, device="cuda", stage=stage)
    fmt = gemm.fmt
    wq, ws = fg8.quantize_weight(w, fmt)
    xq, xs = fg8.quantize_act(x, fmt)
    y = fg8.linear(x, wq, ws, b, fmt).float()
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        xh = _dequant(xq, xs)
        wh = _dequant(wq, ws)
        ref = xh @ wh.t() + b.float()
        bound = xh.abs() @ wh.abs().t()
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    bad = ~((y - ref).abs() <= 8e-3 * bound + 1e-6)
    assert int(bad.sum()) == 0, f"{int(bad.sum())} of {bad.numel()} elements out of tolerance"
