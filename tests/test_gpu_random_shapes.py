"""Seeded sweeps of random layer shapes through every entry point vs the CPU oracle.

The fixed-shape tests pin each kernel path on hand-picked sizes; this sweep
draws M, N and K at random inside each path's range, in both scale formats and
at weight blocks 128, 64 and 32, so that the dispatch rule, the tile and
K-block edges, the split-K tail plans and the few-token split counts meet
shapes nobody chose.  Each case is checked within the y tolerance on every row
(small M) or on sampled rows that always include the first and last row and
the 128-row tile boundaries, the weight codes are compared with the oracle's
bit for bit, and a second call must give the same bits.  A CPU test checks
that the drawn shapes really reach every path fg8_linear_plan reports
(tiled with and without a split tail, the few-token kernel, the fused
few-token kernel).  The same kind of draw runs the two-layer chain (the
epilogue's requantized codes and scales bit-exact against the oracle's
quantization of the stored output), the in-launch quantization, the static
activation scale, the MoE expert GEMM on random routing, and the
quantizers themselves (strided rows, blocks 128/64/32, codes and scales bit
for bit, and Fp8Dequantize back).  A last set takes M, N and K on and next
to the tile, block and path boundaries and checks every element.
"""
import numpy as np
import pytest
import torch

import workloads as W
from _ws_layout import decode
from conftest import y_tolerance

FLOAT, UE8M0 = 0, 1


def _cases():
    """(name, M, N, K, fmt, block, bias): N a multiple of 8 and K of 16 (the
    rows' 16-byte alignment the boundary asks for), everything else free."""
    rng = np.random.default_rng(20261203)
    out = []

    def draw(kind, n, m_lo, m_hi, n_lo, n_hi, k_lo, k_hi, block=128):
        for i in range(n):
            M = int(rng.integers(m_lo, m_hi + 1))
            N = 8 * int(rng.integers(n_lo // 8, n_hi // 8 + 1))
            K = 16 * int(rng.integers(k_lo // 16, k_hi // 16 + 1))
            fmt = len(out) % 2
            bias = bool(rng.integers(0, 4))  # three in four with a bias
            out.append((f"{kind}{i}", M, N, K, fmt, block, bias))

    draw("few", 32, 1, 32, 8, 3072, 16, 4096)             # few-token kernel (fused for UE8M0 and M <= 16)
    draw("mid", 24, 33, 128, 8, 12288, 16, 2048)           # few-token below the tiled rule, tiled above
    draw("tiled", 32, 129, 1100, 128, 2400, 16, 2560)     # whole tiles, short and long K
    draw("split", 20, 129, 640, 256, 2560, 8192, 10240)    # >= 64 K-blocks: split-K tails
    draw("b64_", 12, 1, 700, 8, 1536, 16, 2048, block=64)
    draw("b32_", 12, 1, 700, 8, 1536, 16, 2048, block=32)
    return out


CASES = _cases()


def test_sweep_reaches_every_path():
    """The drawn shapes reach each kernel fg8_linear_plan can report, in both
    formats (block-128 cases), including split-K tails."""
    from fine_grained_fp8_act_b200 import build
    build.build()
    import fine_grained_fp8_act_b200 as fg8
    seen = set()
    for _, M, N, K, fmt, block, _ in CASES:
        if block != 128:
            continue
        kernel, _, split_tiles, _ = fg8.fg8_linear_plan(M, N, K, fmt)
        seen.add((fmt, kernel, kernel == 0 and split_tiles > 0))
    want = {(FLOAT, 0, False), (FLOAT, 0, True), (FLOAT, 1, False),
            (UE8M0, 0, False), (UE8M0, 0, True), (UE8M0, 2, False)}
    assert want <= seen, sorted(want - seen)


def test_tolerance_admits_the_rounded_output(orc):
    """A bias-dominated layer with few K-elements (shapes the sweep draws):
    the oracle's own correctly rounded bf16 y misses the bound 8e-3 * sum |xhat
    * what| + 1e-6 on some element, and is within it once half a bf16 ulp of y
    (the output format's rounding) is added, which the sweep therefore uses."""
    M, N, K, fmt, block = 309, 1304, 48, UE8M0, 64
    seed = M * 7919 + N * 31 + K
    x = W.x_outliers(M, K, seed=seed)
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1, rows_per_group=block)
    b = W.normal((N,), 0.1, seed=seed + 2)
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt, block)
    y64, bound, ybf = orc.linear(W.bf16_bits(x), owq, ows, W.bf16_bits(b), fmt, block=block)
    rounded = (ybf.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(rounded - y64)
    assert (err > y_tolerance(bound)).any()
    assert (err <= y_tolerance(bound, y64, rounded)).all()


@pytest.fixture(scope="module")
def fg8():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


def _f64(t):
    return (W.bf16_bits(t.cpu()).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rows(M, seed):
    if M <= 48:
        return None
    rng = np.random.default_rng(seed)
    r = {0, M - 1, M // 2} | {b + d for b in range(128, M, 128) for d in (-1, 0) if b + d < M}
    r |= set(int(v) for v in rng.integers(0, M, 16))
    return np.array(sorted(r), dtype=np.int64)


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N,K,fmt,block,bias", CASES, ids=[c[0] for c in CASES])
def test_random_shape_vs_oracle(fg8, orc, name, M, N, K, fmt, block, bias):
    seed = M * 7919 + N * 31 + K
    x = W.x_outliers(M, K, seed=seed)
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1, rows_per_group=block)
    b = W.normal((N,), 0.1, seed=seed + 2) if bias else None
    xd, wd = x.cuda(), w.cuda()
    bd = None if b is None else b.cuda()
    wq, ws = fg8.quantize_weight(wd, fmt, block=block)
    y = fg8.linear(xd, wq, ws, bd, fmt, block=block)
    y_again = fg8.linear(xd, wq, ws, bd, fmt, block=block)
    torch.cuda.synchronize()
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt, block)
    assert np.array_equal(wq.view(torch.uint8).cpu().numpy(), owq), f"{name}: weight codes"
    r = _rows(M, seed)
    y64, bound, _ = orc.linear(W.bf16_bits(x), owq, ows, None if b is None else W.bf16_bits(b), fmt, rows=r,
                               block=block)
    got = _f64(y if r is None else y[torch.from_numpy(r).cuda()])
    err = np.abs(got - y64)
    bad = ~(err <= y_tolerance(bound, y64, got))
    plan = fg8.fg8_linear_plan(M, N, K, fmt) if block == 128 else None
    assert not bad.any(), (f"{name} M={M} N={N} K={K} fmt={fmt} block={block} plan={plan}: "
                           f"{int(bad.sum())} elements out of tolerance, max err {np.nanmax(err)}")
    assert torch.equal(y, y_again), f"{name}: a second call gave other bits"


# ------------------------------------------- chained, fused and static ----
def _entry_cases():
    """Random shapes for the entry points beside fg8_linear: (name, M, K1, N1,
    N2, fmt, bias).  N1 is the next layer's K, so a multiple of 16."""
    rng = np.random.default_rng(4417)
    out = []
    for i in range(24):
        M = int(rng.integers(1, 1101)) if i % 3 else int(rng.integers(1, 40))
        K1 = 16 * int(rng.integers(1, 257))
        N1 = 16 * int(rng.integers(1, 161))
        N2 = 8 * int(rng.integers(1, 241))
        out.append((f"e{i}", M, K1, N1, N2, i % 2, bool(rng.integers(0, 4))))
    return out


ENTRY_CASES = _entry_cases()


def _same(got, want, what):
    got, want = np.ascontiguousarray(got), np.ascontiguousarray(want)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {tuple(bad[0])}")


def _check_y(y, y64, bound, what):
    got = _f64(y)
    err = np.abs(got - y64)
    bad = ~(err <= y_tolerance(bound, y64, got))
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, max err {np.nanmax(err)}"


def _layers(fg8, orc, M, K1, N1, N2, fmt, bias):
    seed = M * 131 + K1 * 7 + N1 * 3 + N2
    x = W.x_outliers(M, K1, seed=seed)
    w1 = W.w_row_groups(N1, K1, 0.02, seed=seed + 1)
    w2 = W.normal((N2, N1), 0.02, seed=seed + 2)
    b1 = W.normal((N1,), 0.1, seed=seed + 3) if bias else None
    wq1, ws1 = fg8.quantize_weight(w1.cuda(), fmt)
    wq2, ws2 = fg8.quantize_weight(w2.cuda(), fmt)
    owq1, ows1 = orc.quantize_weight(W.bf16_bits(w1), fmt)
    owq2, ows2 = orc.quantize_weight(W.bf16_bits(w2), fmt)
    return x, b1, (wq1, ws1, owq1, ows1), (wq2, ws2, owq2, ows2)


def _check_chain(fg8, orc, name, M, N1, N2, fmt, x, b1, y1, wsn, second, rows):
    """y1 vs the oracle; the next layer's codes and scales decoded from its
    workspace vs the oracle's quantization of the stored y1, bit for bit; y2
    (fg8_linear_run from that workspace) vs the oracle on those codes."""
    wq2, ws2, owq2, ows2 = second
    y2 = torch.full((M, N2), float("nan"), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    fg8.fg8_linear_run(wq2.data_ptr(), ws2.data_ptr(), 0, y2.data_ptr(), M, N2, N1, N2, fmt, wsn.data_ptr(),
                       wsn.numel(), s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsn.data_ptr(), s) == 0
    nxq, nxs = decode(wsn.cpu().numpy(), M, N1, fmt)
    oxq, oxs = orc.quantize_act(W.bf16_bits(y1.cpu()), fmt)
    _same(nxq, oxq, f"{name}: requantized codes of y1")
    _same(nxs, oxs.view(np.uint32) if fmt == FLOAT else oxs, f"{name}: requantized scales of y1")
    y2_64, bound2, _ = orc.linear_dequant(oxq, oxs, owq2, ows2, None, fmt, rows=rows)
    _check_y(y2 if rows is None else y2[torch.from_numpy(rows).cuda()], y2_64, bound2, f"{name}: y2")


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K1,N1,N2,fmt,bias", ENTRY_CASES, ids=[c[0] for c in ENTRY_CASES])
def test_random_chain_vs_oracle(fg8, orc, name, M, K1, N1, N2, fmt, bias):
    """fg8_linear_prepare + fg8_linear_run_chain (the epilogue quantizes y1 for
    the next layer) + fg8_linear_run of the next layer."""
    x, b1, first, second = _layers(fg8, orc, M, K1, N1, N2, fmt, bias)
    wq1, ws1, owq1, ows1 = first
    s = torch.cuda.current_stream().cuda_stream
    wsa = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N1, K1, fmt), dtype=torch.uint8, device="cuda")
    wsb = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N2, N1, fmt), dtype=torch.uint8, device="cuda")
    y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
    xd = x.cuda()
    b1d = None if b1 is None else b1.cuda()
    fg8.fg8_linear_prepare(xd.data_ptr(), M, N1, K1, K1, ws1.data_ptr(), fmt, wsa.data_ptr(), wsa.numel(), s)
    fg8.fg8_linear_run_chain(wq1.data_ptr(), ws1.data_ptr(), 0 if b1d is None else b1d.data_ptr(), y1.data_ptr(),
                             M, N1, K1, N1, fmt, wsa.data_ptr(), wsa.numel(), N2, ws2_ptr(second), wsb.data_ptr(),
                             wsb.numel(), s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsa.data_ptr(), s) == 0
    rows = _rows(M, M + K1)
    y1_64, bound1, _ = orc.linear(W.bf16_bits(x), owq1, ows1, None if b1 is None else W.bf16_bits(b1), fmt,
                                  rows=rows)
    _check_y(y1 if rows is None else y1[torch.from_numpy(rows).cuda()], y1_64, bound1, f"{name}: y1")
    _check_chain(fg8, orc, name, M, N1, N2, fmt, x, b1, y1, wsb, second, rows)


def ws2_ptr(second):
    return second[1].data_ptr()


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K1,N1,N2,fmt,bias", ENTRY_CASES, ids=[c[0] for c in ENTRY_CASES])
def test_random_fused_vs_oracle(fg8, orc, name, M, K1, N1, N2, fmt, bias):
    """fg8_linear_fused (x quantized inside the GEMM's launch where the shape
    allows it), with the next layer's quantization on every other case; two
    calls on one workspace give the same bits."""
    x, b1, first, second = _layers(fg8, orc, M, K1, N1, N2, fmt, bias)
    wq1, ws1, owq1, ows1 = first
    s = torch.cuda.current_stream().cuda_stream
    chain = int(name[1:]) % 4 < 2
    wsa = torch.zeros(fg8.fg8_linear_fused_workspace_bytes(M, N1, K1, fmt), dtype=torch.uint8, device="cuda")
    wsb = torch.zeros(fg8.fg8_linear_workspace_bytes(M, N2, N1, fmt), dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    b1d = None if b1 is None else b1.cuda()
    ys = []
    for _ in range(2):
        y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
        fg8.fg8_linear_fused(xd.data_ptr(), M, N1, K1, K1, wq1.data_ptr(), ws1.data_ptr(),
                             0 if b1d is None else b1d.data_ptr(), y1.data_ptr(), N1, fmt, wsa.data_ptr(),
                             wsa.numel(), N2 if chain else 0, ws2_ptr(second) if chain else None,
                             wsb.data_ptr() if chain else None, wsb.numel() if chain else 0, stream=s)
        torch.cuda.synchronize()
        assert fg8.fg8_check_device_status(wsa.data_ptr(), s) == 0
        ys.append(y1)
    assert torch.equal(ys[0], ys[1]), f"{name}: a second call gave other bits"
    y1 = ys[1]
    rows = _rows(M, M + K1)
    y1_64, bound1, _ = orc.linear(W.bf16_bits(x), owq1, ows1, None if b1 is None else W.bf16_bits(b1), fmt,
                                  rows=rows)
    _check_y(y1 if rows is None else y1[torch.from_numpy(rows).cuda()], y1_64, bound1, f"{name}: y1")
    if chain:
        _check_chain(fg8, orc, name, M, N1, N2, fmt, x, b1, y1, wsb, second, rows)


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K1,N1,N2,fmt,bias", ENTRY_CASES[::2], ids=[c[0] for c in ENTRY_CASES[::2]])
def test_random_static_vs_oracle(fg8, orc, name, M, K1, N1, N2, fmt, bias):
    """fg8_linear_static (one precomputed activation scale, float weight
    scales) on the same random shapes."""
    x, b1, first, _ = _layers(fg8, orc, M, K1, N1, N2, FLOAT, bias)
    wq1, ws1, owq1, ows1 = first
    scale = float(np.float32(3.0 / 448.0))  # the 20x outlier channels saturate
    st = torch.tensor([scale], dtype=torch.float32, device="cuda")
    y1 = fg8.linear_static(x.cuda(), st, wq1, ws1, None if b1 is None else b1.cuda())
    torch.cuda.synchronize()
    oq, oxs = orc.quantize_act_static(W.bf16_bits(x), scale)
    rows = _rows(M, M + K1)
    y64, bound, _ = orc.linear_dequant(oq, oxs, owq1, ows1, None if b1 is None else W.bf16_bits(b1), FLOAT,
                                       rows=rows)
    _check_y(y1 if rows is None else y1[torch.from_numpy(rows).cuda()], y64, bound, f"{name}: y")


# ----------------------------------------------------------- MoE experts ----
def _grouped_cases():
    """(name, T tokens, E experts, topk, K, N, fmt, skew, bias)."""
    rng = np.random.default_rng(977)
    out = []
    for i in range(12):
        E = int(rng.integers(1, 13))
        out.append((f"g{i}", int(rng.integers(1, 257)), E, int(rng.integers(1, min(E, 4) + 1)),
                    16 * int(rng.integers(1, 65)), 8 * int(rng.integers(1, 65)), i % 2,
                    float(rng.uniform(0.3, 2.0)), bool(rng.integers(0, 4))))
    return out


GROUPED_CASES = _grouped_cases()


@pytest.mark.gpu
@pytest.mark.parametrize("name,T,E,topk,K,N,fmt,skew,bias", GROUPED_CASES, ids=[c[0] for c in GROUPED_CASES])
def test_random_grouped_vs_oracle(fg8, orc, name, T, E, topk, K, N, fmt, skew, bias):
    """fg8_grouped_linear on random routing (log-normal expert popularity,
    padded expert runs) and random shapes: every written row vs the oracle,
    the padding blocks' rows left untouched."""
    seed = T * 17 + E * 5 + K + N
    rt, re = W.moe_routing(T, E, topk, seed=seed, skew=skew)
    x = W.gather_rows(W.x_outliers(T, K, seed=seed + 1), rt)
    M = x.shape[0]
    ws_bf16 = [W.w_row_groups(N, K, 0.02, seed=seed + 10 + e) for e in range(E)]
    qs = [fg8.quantize_weight(w.cuda(), fmt) for w in ws_bf16]
    wq = torch.stack([q.view(torch.uint8) for q, _ in qs])
    ws = torch.stack([s if s.element_size() != 1 else s.view(torch.uint8) for _, s in qs])
    b = W.normal((E, N), 0.1, seed=seed + 2) if bias else None
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nb = fg8.fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    xd, red = x.cuda(), re.cuda()
    bd = None if b is None else b.cuda()
    fg8.fg8_grouped_linear(xd.data_ptr(), M, K, K, red.data_ptr(), E, N, wq.data_ptr(), ws.data_ptr(),
                           0 if bd is None else bd.data_ptr(), y.data_ptr(), N, fmt, wsp.data_ptr(), nb, s)
    torch.cuda.synchronize()
    assert fg8.fg8_check_device_status(wsp.data_ptr(), s) == 0
    y64, bound, _, written = orc.grouped_linear(W.bf16_bits(x), re.numpy(), wq.cpu().numpy(), ws.cpu().numpy(),
                                                None if b is None else W.bf16_bits(b), fmt)
    got = _f64(y)
    assert np.isnan(got[~written]).all(), f"{name}: rows of skipped blocks were written"
    assert written[re.numpy() >= 0].all()
    err = np.abs(got[written] - y64[written])
    bad = ~(err <= y_tolerance(bound[written], y64[written], got[written]))
    assert not bad.any(), f"{name} M={M} E={E} K={K} N={N} fmt={fmt}: {int(bad.sum())} out of tolerance"


# ----------------------------------------------------------- quantizers ----
def _quant_cases():
    """(name, rows, cols, pad, fmt, block): pad extra bf16 columns per row of
    the input's allocation (a strided view), a multiple of 8."""
    rng = np.random.default_rng(5311)
    return [(f"q{i}", int(rng.integers(1, 3000)), 16 * int(rng.integers(1, 400)), 8 * int(rng.integers(0, 3)),
             i % 2, (128, 64, 32)[i % 3]) for i in range(18)]


QUANT_CASES = _quant_cases()


def _scale_bits(s):
    """Scales as bit patterns: float32 as uint32, UE8M0 bytes as they are."""
    if isinstance(s, torch.Tensor):
        s = (s.view(torch.uint8) if s.element_size() == 1 else s).cpu().numpy()
    return s.view(np.uint32) if s.dtype == np.float32 else s


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K,pad,fmt,block", QUANT_CASES, ids=[c[0] for c in QUANT_CASES])
def test_random_quantizers_bits(fg8, orc, name, M, K, pad, fmt, block):
    """Activation and weight quantization of random shapes (strided rows for
    x), codes and scales bit for bit against the oracle; block 128 weights
    also back through Fp8Dequantize, bit for bit."""
    wide = W.x_outliers(M, K + pad, seed=M + K + pad)
    x = wide.cuda()[:, :K]
    xq, xs = fg8.quantize_act(x, fmt, block=block)
    wq, ws = fg8.quantize_weight(x, fmt, block=block)  # the same matrix as a weight [N = M, K]
    torch.cuda.synchronize()
    bits = W.bf16_bits(wide[:, :K].contiguous())
    oq, oxs = orc.quantize_act(bits, fmt, block)
    owq, ows = orc.quantize_weight(bits, fmt, block)
    _same(xq.view(torch.uint8).cpu().numpy(), oq, f"{name}: activation codes")
    _same(_scale_bits(xs), _scale_bits(oxs), f"{name}: activation scales")
    _same(wq.view(torch.uint8).cpu().numpy(), owq, f"{name}: weight codes")
    _same(_scale_bits(ws), _scale_bits(ows), f"{name}: weight scales")
    if block == 128:
        wd = fg8.dequantize_weight(wq, ws, fmt)
        torch.cuda.synchronize()
        _same(W.bf16_bits(wd.cpu()), orc.dequantize_weight(owq, ows, fmt), f"{name}: dequantized weight")


# ----------------------------------------------------- boundary values ----
def _edge_cases():
    """Shapes whose M, N and K sit on or next to a tile, block or path
    boundary (the few-token limits 16 / 32 / 128, the 128-row tile, the
    128- and 256-column tiles, the 128-channel group), a seeded subset of
    their product, both formats."""
    Ms = [1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 255, 257, 383]
    Ns = [8, 120, 128, 136, 248, 256, 264, 1016, 1024, 1032]
    Ks = [16, 112, 128, 144, 240, 256, 272, 1024, 4080, 4112]
    rng = np.random.default_rng(8128)
    combos = [(m, n, k) for m in Ms for n in Ns for k in Ks]
    pick = rng.choice(len(combos), size=64, replace=False)
    return [(f"edge{i}", *combos[j], i % 2) for i, j in enumerate(sorted(pick))]


EDGE_CASES = _edge_cases()


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,N,K,fmt", EDGE_CASES, ids=[c[0] for c in EDGE_CASES])
def test_edge_shape_vs_oracle(fg8, orc, name, M, N, K, fmt):
    """Every element against the oracle (these shapes are small)."""
    seed = M * 977 + N * 13 + K
    x = W.x_outliers(M, K, seed=seed)
    w = W.w_row_groups(N, K, 0.02, seed=seed + 1)
    b = W.normal((N,), 0.1, seed=seed + 2)
    wq, ws = fg8.quantize_weight(w.cuda(), fmt)
    y = fg8.linear(x.cuda(), wq, ws, b.cuda(), fmt)
    torch.cuda.synchronize()
    owq, ows = orc.quantize_weight(W.bf16_bits(w), fmt)
    assert np.array_equal(wq.view(torch.uint8).cpu().numpy(), owq), f"{name}: weight codes"
    y64, bound, _ = orc.linear(W.bf16_bits(x), owq, ows, W.bf16_bits(b), fmt)
    _check_y(y, y64, bound, f"{name} M={M} N={N} K={K} fmt={fmt} plan={fg8.fg8_linear_plan(M, N, K, fmt)}")
