"""Guard bands around every output and workspace (the race / out-of-bounds
check in place of a sanitizer): each entry point writes into a region with
4 KiB of a byte pattern before and after it, row-strided outputs keep the
pattern in their padding columns, and a grouped layer's skipped blocks keep
it in their rows.  After the call, all of that must be unchanged and the
written part must equal what the plain call returns."""
import pytest
import torch

import workloads as W
from _canary import Canary

pytestmark = pytest.mark.gpu

FLOAT, UE8M0 = 0, 1
U8, BF16, F32 = torch.uint8, torch.bfloat16, torch.float32


@pytest.fixture(scope="module")
def fg8():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


def _s():
    return torch.cuda.current_stream().cuda_stream


def _sdt(fmt):
    return F32 if fmt == FLOAT else U8


def _bytes(t):
    return t.view(U8) if t.element_size() == 1 else t


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_quantizers_stay_in_bounds(fg8, fmt):
    M, N, K = 129, 264, 400
    Kb, Nb = 4, 3
    x = W.x_outliers(M, K, seed=1).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=2).cuda()
    es = 4 if fmt == FLOAT else 1
    cq, cs = Canary(M * K, "cuda"), Canary(M * Kb * es, "cuda")
    xq, xs = cq.matrix(U8, M, K, K), cs.matrix(_sdt(fmt), M, Kb, Kb)
    fg8.fg8_quantize_act(x.data_ptr(), M, K, K, cq.ptr(), cs.ptr(), fmt, _s())
    wq_c, ws_c = Canary(N * K, "cuda"), Canary(Nb * Kb * es, "cuda")
    wq, ws = wq_c.matrix(U8, N, K, K), ws_c.matrix(_sdt(fmt), Nb, Kb, Kb)
    fg8.fg8_quantize_weight(w.data_ptr(), N, K, K, wq_c.ptr(), ws_c.ptr(), fmt, _s())
    torch.cuda.synchronize()
    rq, rs = fg8.quantize_act(x, fmt)
    rwq, rws = fg8.quantize_weight(w, fmt)
    assert torch.equal(xq, _bytes(rq)) and torch.equal(xs, _bytes(rs))
    assert torch.equal(wq, _bytes(rwq)) and torch.equal(ws, _bytes(rws))
    assert cq.intact() and cs.intact() and wq_c.intact() and ws_c.intact()


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(3, 264, 400), (5, 264, 400), (40, 264, 400), (300, 264, 400),
                                   (5, 1032, 16384), (24, 4104, 2432)])
# fused few-token (UE8M0), few-token, few-token, tiled; few-token with long K / many tiles
def test_linear_stays_in_bounds(fg8, fmt, M, N, K):
    ld_y = N + 8
    x = W.x_outliers(M, K, seed=M).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=M + 1).cuda()
    b = W.normal((N,), 0.1, seed=M + 2).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    cy = Canary(M * ld_y * 2, "cuda")
    y = cy.matrix(BF16, M, N, ld_y)
    need = fg8.fg8_linear_workspace_bytes(M, N, K, fmt)
    cw = Canary(need, "cuda")
    cw.zeroed()
    fg8.fg8_linear(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), b.data_ptr(), cy.ptr(), ld_y, fmt,
                   cw.ptr(), need, _s())
    assert fg8.fg8_check_device_status(cw.ptr(), _s()) == 0
    torch.cuda.synchronize()
    assert torch.equal(y, fg8.linear(x, wq, ws, b, fmt))
    assert cy.intact(), "y: a write outside [M, N] or into the row padding"
    assert cw.intact(), "workspace: a write past fg8_linear_workspace_bytes"


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_grouped_linear_stays_in_bounds(fg8, fmt):
    E, N, K = 3, 264, 400
    M = 3 * 128 + 40
    ld_y = N + 8
    x = W.x_student_t(M, K, seed=5).cuda()
    qs = [fg8.quantize_weight(W.w_row_groups(N, K, 0.02, seed=10 + e).cuda(), fmt) for e in range(E)]
    wq = torch.stack([q.view(U8) for q, _ in qs]).view(qs[0][0].dtype)
    ws = torch.stack([_bytes(s) for _, s in qs]).view(qs[0][1].dtype)
    b = W.normal((E, N), 0.1, seed=6).cuda()
    experts = [1, -1, 0, 2]  # block 1 skipped: its rows must keep the pattern
    re = torch.tensor([experts[r // 128] for r in range(M)], dtype=torch.int32, device="cuda")
    cy = Canary(M * ld_y * 2, "cuda")
    y = cy.matrix(BF16, M, N, ld_y)
    cy.writable[128 * ld_y * 2:256 * ld_y * 2] = False
    need = fg8.fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt)
    cw = Canary(need, "cuda")
    cw.zeroed()
    fg8.fg8_grouped_linear(x.data_ptr(), M, K, K, re.data_ptr(), E, N, wq.data_ptr(), ws.data_ptr(), b.data_ptr(),
                           cy.ptr(), ld_y, fmt, cw.ptr(), need, _s())
    assert fg8.fg8_check_device_status(cw.ptr(), _s()) == 0
    torch.cuda.synchronize()
    ref = fg8.grouped_linear(x, re, wq, ws, b, fmt)
    rows = torch.tensor([r for r in range(M) if experts[r // 128] >= 0], device="cuda")
    assert torch.equal(y[rows], ref[rows])
    assert cy.intact(), "y: a write outside the computed blocks' rows or into the row padding"
    assert cw.intact(), "workspace: a write past fg8_grouped_linear_workspace_bytes"


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_dequantize_stays_in_bounds(fg8, fmt):
    N, K = 300, 400
    ld_w = K + 16
    wq, ws = fg8.quantize_weight(W.normal((N, K), 0.05, seed=7).cuda(), fmt)
    cw = Canary(N * ld_w * 2, "cuda")
    out = cw.matrix(BF16, N, K, ld_w)
    fg8.fg8_dequantize_weight(wq.data_ptr(), N, K, ws.data_ptr(), fmt, cw.ptr(), ld_w, _s())
    torch.cuda.synchronize()
    assert torch.equal(out, fg8.dequantize_weight(wq, ws, fmt))
    assert cw.intact()


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(256, 2048, 8192), (300, 1032, 8192)])  # every tile split over K (ragged too)
def test_split_tail_stays_in_bounds(fg8, fmt, M, N, K):
    plan = fg8.fg8_linear_plan(M, N, K, fmt)
    assert plan[2] > 0 and plan[3] >= 2, plan
    ld_y = N + 8
    x = W.x_outliers(M, K, seed=M + 11).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=M + 12).cuda()
    b = W.normal((N,), 0.1, seed=M + 13).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    cy = Canary(M * ld_y * 2, "cuda")
    y = cy.matrix(BF16, M, N, ld_y)
    need = fg8.fg8_linear_workspace_bytes(M, N, K, fmt)
    cw = Canary(need, "cuda")
    cw.zeroed()
    for _ in range(2):  # the split counters are back at zero for the second call
        fg8.fg8_linear(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), b.data_ptr(), cy.ptr(), ld_y, fmt,
                       cw.ptr(), need, _s())
        assert fg8.fg8_check_device_status(cw.ptr(), _s()) == 0
        torch.cuda.synchronize()
        assert torch.equal(y, fg8.linear(x, wq, ws, b, fmt))
        assert cy.intact(), "y: a write outside [M, N] or into the row padding"
        assert cw.intact(), "workspace: a write past fg8_linear_workspace_bytes (split-K partials included)"


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M", [5, 300])   # few-token kernel quantizing x itself; tiled GEMM quantizing in-launch
def test_fused_linear_stays_in_bounds(fg8, fmt, M):
    N, K = 264, 400
    ld_y = N + 8
    x = W.x_outliers(M, K, seed=M + 3).cuda()
    w = W.w_row_groups(N, K, 0.02, seed=M + 4).cuda()
    b = W.normal((N,), 0.1, seed=M + 5).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    cy = Canary(M * ld_y * 2, "cuda")
    y = cy.matrix(BF16, M, N, ld_y)
    need = fg8.fg8_linear_fused_workspace_bytes(M, N, K, fmt)
    cw = Canary(need, "cuda")
    cw.zeroed()
    for _ in range(2):  # a second call on the same workspace: the flags' epoch has advanced
        fg8.fg8_linear_fused(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), b.data_ptr(), cy.ptr(), ld_y,
                             fmt, cw.ptr(), need, stream=_s())
        assert fg8.fg8_check_device_status(cw.ptr(), _s()) == 0
        torch.cuda.synchronize()
        assert torch.equal(y, fg8.linear(x, wq, ws, b, fmt))
        assert cy.intact(), "y: a write outside [M, N] or into the row padding"
        assert cw.intact(), "workspace: a write past fg8_linear_fused_workspace_bytes"


@pytest.mark.parametrize("blk,sfmt", [(32, "ue8m0"), (64, "ue8m0"), (32, "float"), (64, "float")])
def test_small_block_layer_stays_in_bounds(fg8, blk, sfmt):
    fmt = UE8M0 if sfmt == "ue8m0" else 0
    M, N, K = 200, 264, 400
    ld_y = N + 8
    x = W.x_student_t(M, K, seed=8).cuda()
    b = W.normal((N,), 0.1, seed=9).cuda()
    wq, ws = fg8.quantize_weight(W.w_row_groups(N, K, 0.02, seed=10).cuda(), sfmt, block=blk)
    cy = Canary(M * ld_y * 2, "cuda")
    y = cy.matrix(BF16, M, N, ld_y)
    need = fg8.fg8_linear_block_workspace_bytes(M, N, K, fmt, blk)
    cw = Canary(need, "cuda")
    cw.zeroed()
    fg8.fg8_linear_block(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), b.data_ptr(), cy.ptr(), ld_y,
                         fmt, blk, cw.ptr(), need, _s())
    assert fg8.fg8_check_device_status(cw.ptr(), _s()) == 0
    torch.cuda.synchronize()
    assert torch.equal(y, fg8.linear(x, wq, ws, b, sfmt, block=blk))
    assert cy.intact() and cw.intact()
