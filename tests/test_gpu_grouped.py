"""fg8_grouped_linear -- the MoE expert GEMM on the contiguous grouped layout
-- against the oracle on every written element: seeded skewed routing,
both scale formats, ragged N and K, bias or none, blocks skipped by -1, an
out-of-range expert (reported, its block skipped), and one expert over all
blocks giving the dense layer's bits."""
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


def _expert_stack(fg8, ws_bf16, fmt):
    """[E, N, K] e4m3 weights and [E, Nb, Kb] scales, each expert quantized on
    its own (same dtypes as fg8.quantize_weight returns: a bit copy)."""
    qs = [fg8.quantize_weight(w, fmt) for w in ws_bf16]

    def stack(ts):  # stacked as bytes (no float8 arithmetic involved), viewed back
        if ts[0].element_size() != 1:
            return torch.stack(ts)
        return torch.stack([t.view(torch.uint8) for t in ts]).view(ts[0].dtype)
    return stack([q for q, _ in qs]), stack([s for _, s in qs])


def _u8(t):
    """Bytes of a float8 tensor (or the float32 scales as they are) for the oracle."""
    return (t.view(torch.uint8) if t.element_size() == 1 else t).cpu().numpy()


def _case(fg8, T, E, topk, K, N, fmt, seed, bias=True):
    rt, re = W.moe_routing(T, E, topk, seed=seed, skew=1.0)
    xt = W.x_outliers(T, K, seed=seed + 1).cuda()
    x = W.gather_rows(xt, rt)
    wq, ws = _expert_stack(fg8, [W.w_row_groups(N, K, 0.02, seed=seed + 10 + e).cuda() for e in range(E)], fmt)
    b = W.normal((E, N), 0.1, seed=seed + 2).cuda() if bias else None
    return x, re.cuda(), wq, ws, b


def _run(fg8, x, re, wq, ws, b, fmt):
    M = x.shape[0]
    E, N, K = wq.shape
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    nb = fg8.fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    fg8.fg8_grouped_linear(x.data_ptr(), M, K, x.stride(0), re.data_ptr(), E, N, wq.data_ptr(), ws.data_ptr(),
                           0 if b is None else b.data_ptr(), y.data_ptr(), N, fmt, wsp.data_ptr(), nb, s)
    st = fg8.fg8_check_device_status(wsp.data_ptr(), s)
    return y, st


def _check(orc, x, re, wq, ws, b, y, fmt):
    bits = W.bf16_bits
    y64, bound, _, written = orc.grouped_linear(bits(x), re.cpu().numpy(), _u8(wq), _u8(ws),
                                                None if b is None else bits(b), fmt)
    yb = bits(y)
    yg = (yb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.isnan(yg[~written]).all(), "rows of skipped blocks were written"
    err = np.abs(yg[written] - y64[written])
    tol = y_tolerance(bound[written])
    bad = ~(err <= tol)  # NaN counts as out of tolerance
    assert not bad.any(), f"{bad.sum()} of {bad.size} out of tolerance; worst {np.nanmax(err - tol)}"
    return written


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("T,E,topk,K,N", [(300, 6, 2, 512, 384), (200, 5, 3, 400, 264), (90, 9, 4, 1024, 136)])
def test_grouped_vs_oracle(fg8, orc, fmt, T, E, topk, K, N):
    x, re, wq, ws, b = _case(fg8, T, E, topk, K, N, fmt, seed=T + E)
    y, st = _run(fg8, x, re, wq, ws, b, fmt)
    assert st == 0
    written = _check(orc, x, re, wq, ws, b, y, fmt)
    assert written[(re.cpu().numpy() >= 0)].all()


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_grouped_skipped_blocks_and_no_bias(fg8, orc, fmt):
    x, re, wq, ws, _ = _case(fg8, 400, 4, 2, 256, 256, fmt, seed=41, bias=False)
    re = re.clone()
    re[128] = -1  # the second block is skipped as a whole
    y, st = _run(fg8, x, re, wq, ws, None, fmt)
    assert st == 0
    written = _check(orc, x, re, wq, ws, None, y, fmt)
    assert not written[128:256].any()


def test_grouped_unknown_expert_is_reported(fg8, orc):
    x, re, wq, ws, b = _case(fg8, 300, 4, 2, 256, 128, UE8M0, seed=51)
    re = re.clone()
    re[256] = 4  # == E: that block is skipped and the status word says so
    y, st = _run(fg8, x, re, wq, ws, b, UE8M0)
    assert st == fg8.FG8_ERR_INVALID_ARG
    re_ok = re.clone()
    re_ok[256] = -1
    _check(orc, x, re_ok, wq, ws, b, y, UE8M0)


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_one_expert_is_the_dense_layer(fg8, fmt):
    """Every block on expert 0: the dense fg8_linear's bits (tiled GEMM)."""
    M, K, N = 640, 768, 520
    x = W.x_student_t(M, K, seed=61).cuda()
    w = W.normal((N, K), 0.02, seed=62).cuda()
    b = W.normal((N,), 0.1, seed=63).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    y_dense = fg8.linear(x, wq, ws, b, "ue8m0" if fmt else "float")
    re = torch.zeros(M, dtype=torch.int32, device="cuda")
    y, st = _run(fg8, x, re, wq[None].contiguous(), ws[None].contiguous(), b[None].contiguous(), fmt)
    assert st == 0
    assert torch.equal(y, y_dense)


def test_layer_wrapper(fg8, orc):
    x, re, wq, ws, b = _case(fg8, 150, 3, 2, 256, 256, UE8M0, seed=71)
    y = fg8.grouped_linear(x, re, wq, ws, b, "ue8m0")
    torch.cuda.synchronize()
    y2, st = _run(fg8, x, re, wq, ws, b, UE8M0)
    assert st == 0
    written = _check(orc, x, re, wq, ws, b, y2, UE8M0)
    assert torch.equal(y[torch.from_numpy(written).cuda()], y2[torch.from_numpy(written).cuda()])


def test_moe_full_size_sampled(fg8, orc):
    """The bench's MoE gate/up layer at full size (4096 tokens x top-8 on 256
    experts, K = 7168 -> N = 4096, UE8M0) in the bench's launch
    configuration; sampled rows of several blocks (first, middle, last routed
    row) checked on every column against the oracle with the block's expert."""
    c = W.DSV3_MOE
    E, K, N = c["experts"], c["hidden"], 2 * c["inter"]
    rt, re = W.moe_routing(c["tokens"], E, c["topk"], seed=5, skew=c["skew"])
    x = W.gather_rows(W.x_student_t(c["tokens"], K, seed=50, device="cuda"), rt)
    M = x.shape[0]
    wq = torch.empty(E, N, K, dtype=torch.float8_e4m3fn, device="cuda")
    ws = torch.empty(E, N // 128, K // 128, dtype=torch.float8_e8m0fnu, device="cuda")
    for e in range(E):
        q, s = fg8.quantize_weight(W.w_row_groups(N, K, 0.015, seed=1000 + e, device="cuda"), UE8M0)
        wq[e] = q
        ws[e] = s
    re_d = re.cuda()
    y, st = _run(fg8, x, re_d, wq, ws, None, UE8M0)
    assert st == 0
    blocks = M // 128
    heads = re.view(-1, 128)[:, 0]
    for t in sorted({0, 1, blocks // 2, blocks - 1}):
        e = int(heads[t])
        real = (re[t * 128:(t + 1) * 128] >= 0).nonzero().flatten()
        rows = t * 128 + torch.unique(torch.stack([real[0], real[len(real) // 2], real[-1]]))
        xb = W.bf16_bits(x[rows])
        y64, bound, _, written = orc.grouped_linear(xb, np.zeros(len(rows), np.int32), _u8(wq[e:e + 1]),
                                                    _u8(ws[e:e + 1]), None, UE8M0)
        yg = (W.bf16_bits(y[rows]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        err = np.abs(yg - y64)
        assert written.all() and (err <= y_tolerance(bound)).all(), f"block {t} (expert {e})"


def test_batched_layout(fg8, orc):
    """The batched layout (E slabs of cap rows, counts[e] routed) through
    fg8_grouped_row_expert and the grouped GEMM: the index matches its
    definition, empty and partial slabs skip their trailing blocks."""
    E, cap, K, N = 4, 256, 256, 136
    counts = torch.tensor([0, 130, 300, 5], dtype=torch.int32, device="cuda")
    re = torch.full((E * cap,), 7, dtype=torch.int32, device="cuda")
    fg8.fg8_grouped_row_expert(counts.data_ptr(), E, cap, re.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    want = np.concatenate([np.where(np.arange(cap) < c, e, -1) for e, c in enumerate(counts.tolist())])
    assert np.array_equal(re.cpu().numpy(), want.astype(np.int32))
    x = W.x_normal(E * cap, K, seed=81).cuda()
    wq, ws = _expert_stack(fg8, [W.normal((N, K), 0.02, seed=82 + e).cuda() for e in range(E)], UE8M0)
    y, st = _run(fg8, x, re, wq, ws, None, UE8M0)
    assert st == 0
    written = _check(orc, x, re, wq, ws, None, y, UE8M0)
    assert written.sum() == 0 + 256 + 256 + 128  # the blocks whose first row is routed
