"""The tiled GEMM's split-K tail vs the CPU oracle.

When the tiles do not fill a whole number of waves over the SMs, the tiles of
the last, partial wave are each split over K into units that run on the
otherwise idle SMs; every unit writes its fp32 partial sum and the tile's
last unit adds them in split order, applies the bias and stores the tile
(and, in a chain, quantizes it for the next layer).  These shapes are chosen
so that the plan splits: one with every tile split (fewer tiles than SMs),
others with whole tiles followed by a split tail, with ragged M, N and K.
Outputs are compared with the oracle within the y tolerance (all of them,
or every row of the split tiles plus sampled rows); repeated calls and the
entry points that share the plan give the same bits.
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


def _f64(t):
    return (W.bf16_bits(t.cpu()).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(y, y64, bound, what):
    err = np.abs(_f64(y) - y64)
    bad = ~(err <= y_tolerance(bound))
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, max err {np.nanmax(err)}"


def _scale_bits(s, fmt):
    return s.view(np.uint32) if fmt == FLOAT else s


def _rows(M, split_rows, n=40, seed=0):
    """Sampled output rows: every row of the split tiles' row blocks in
    `split_rows`, tile boundaries, and random others."""
    rng = np.random.default_rng(seed)
    base = {0, 127, 128, M - 1, M // 2} | set(int(r) for r in rng.integers(0, M, n))
    return np.array(sorted(base | set(split_rows)), dtype=np.int64)


# (M, N, K, rows to check, or None for all): fewer tiles than SMs, every tile
# split (32 tiles of 128 x 128, 64 K-blocks); whole tiles then a split tail
# (160 tiles of 128 x 256 on 148 SMs; the last 12, row blocks 16-19, are
# split); the same with a ragged M, N and K (K-blocks 64, the last 96 wide)
SHAPES = [(256, 2048, 8192, None), (2560, 2048, 8192, range(2048, 2560)),
          (2500, 2040, 8160, range(2048, 2500))]


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K,rows", SHAPES)
def test_split_tail_vs_oracle(fg8, orc, fmt, M, N, K, rows):
    plan = fg8.fg8_linear_plan(M, N, K, fmt)
    assert plan[0] == 0 and plan[2] > 0 and plan[3] >= 2, plan  # the shape does split
    x = W.x_outliers(M, K, seed=M + K)
    w = W.w_row_groups(N, K, 0.02, seed=N + K)
    b = W.normal((N,), 0.1, seed=N)
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    wq, ws = fg8.quantize_weight(wd, fmt)
    y = fg8.linear(xd, wq, ws, bd, fmt)
    y_again = fg8.linear(xd, wq, ws, bd, fmt)
    torch.cuda.synchronize()
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
    assert np.array_equal(wq.view(torch.uint8).cpu().numpy(), owq)
    r = None if rows is None else _rows(M, rows, seed=M)
    y64, bound, _ = orc.linear(W.bf16_bits(x), owq, ows, W.bf16_bits(b), fmt, rows=r)
    _check(y if r is None else y[torch.from_numpy(r).cuda()], y64, bound, f"M={M} N={N} K={K} fmt={fmt}")
    assert torch.equal(y, y_again), "the split sums depend on which unit finished last"
    # the pre-quantized GEMM and the in-launch quantization plan the same split
    xq, xs = fg8.quantize_act(xd, fmt)
    assert torch.equal(fg8.gemm_prequant(xq, xs, wq, ws, bd, fmt), y)
    nb = fg8.fg8_linear_fused_workspace_bytes(M, N, K, fmt)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    yf = torch.empty_like(y)
    s = torch.cuda.current_stream().cuda_stream
    fg8.fg8_linear_fused(xd.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), bd.data_ptr(), yf.data_ptr(), N,
                         fmt, wsp.data_ptr(), nb, stream=s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsp.data_ptr(), s) == 0
    assert torch.equal(yf, y)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_split_tail_in_a_chain(fg8, orc, fmt):
    """A chained layer whose last wave is split: the tile's last unit also
    quantizes y for the next layer, bit-exact against the oracle's
    quantization of the stored y."""
    M, K1, N1, N2 = 700, 8192, 6512, 264  # 156 tiles of 128 x 256: the last 8 split; N1 = the next layer's K
    x = W.x_student_t(M, K1, seed=5)
    w1 = W.normal((N1, K1), 0.02, seed=6)
    w2 = W.w_row_groups(N2, N1, 0.02, seed=7)
    b1 = W.normal((N1,), 0.1, seed=8)
    xd, w1d, w2d, b1d = x.cuda(), w1.cuda(), w2.cuda(), b1.cuda()
    wq1, ws1 = fg8.quantize_weight(w1d, fmt)
    wq2, ws2 = fg8.quantize_weight(w2d, fmt)
    s = torch.cuda.current_stream().cuda_stream
    wsa = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N1, K1, fmt), dtype=torch.uint8, device="cuda")
    wsb = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N2, N1, fmt), dtype=torch.uint8, device="cuda")
    y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
    y2 = torch.full((M, N2), float("nan"), dtype=torch.bfloat16, device="cuda")
    fg8.fg8_linear_prepare(xd.data_ptr(), M, N1, K1, K1, ws1.data_ptr(), fmt, wsa.data_ptr(), wsa.numel(), s)
    fg8.fg8_linear_run_chain(wq1.data_ptr(), ws1.data_ptr(), b1d.data_ptr(), y1.data_ptr(), M, N1, K1, N1, fmt,
                             wsa.data_ptr(), wsa.numel(), N2, ws2.data_ptr(), wsb.data_ptr(), wsb.numel(), s)
    torch.cuda.synchronize()
    nxq, nxs = decode(wsb.cpu().numpy(), M, N1, fmt)
    fg8.fg8_linear_run(wq2.data_ptr(), ws2.data_ptr(), 0, y2.data_ptr(), M, N2, N1, N2, fmt, wsb.data_ptr(),
                       wsb.numel(), s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsa.data_ptr(), s) == 0
    assert fg8.fg8_check_device_status(wsb.data_ptr(), s) == 0
    owq1, ows1 = orc.quantize_weight(W.bf16_bits(w1), fmt)
    owq2, ows2 = orc.quantize_weight(W.bf16_bits(w2), fmt)
    # y1 on every row of two row blocks (the split tiles span all six row
    # blocks, in column blocks 24-25) and sampled others
    r = _rows(M, list(range(0, 128)) + list(range(640, 700)), seed=3)
    y1_64, bound1, _ = orc.linear(W.bf16_bits(x), owq1, ows1, W.bf16_bits(b1), fmt, rows=r)
    _check(y1[torch.from_numpy(r).cuda()], y1_64, bound1, "y1")
    oxq, oxs = orc.quantize_act(W.bf16_bits(y1.cpu()), fmt)
    assert np.array_equal(np.ascontiguousarray(nxq), oxq), "requantized codes of y1"
    assert np.array_equal(np.ascontiguousarray(nxs), _scale_bits(oxs, fmt)), "requantized scales of y1"
    y2_64, bound2, _ = orc.linear_dequant(oxq, oxs, owq2, ows2, None, fmt)
    _check(y2, y2_64, bound2, "y2")
