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
