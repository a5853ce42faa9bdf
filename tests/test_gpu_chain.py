"""Two chained layers (fg8_linear_run_chain): the first layer's GEMM epilogue
quantizes its bf16 output for the second layer.  Both outputs must equal,
bit for bit, what two separate fg8_linear calls produce (which the other GPU
tests check against the oracle)."""
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


def _ws(fg8, M, N, K, fmt):
    return torch.zeros(fg8.fg8_linear_workspace_bytes(M, N, K, fmt), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K1,N1,N2", [(8176, 480, 1920, 480), (300, 256, 528, 136), (129, 144, 1040, 264),
                                        (1, 128, 256, 16), (640, 1024, 4096, 1024)])
def test_chain_equals_two_layers(fg8, fmt, M, K1, N1, N2):
    x = W.x_outliers(M, K1, seed=M + K1).cuda()
    w1 = W.normal((N1, K1), 0.02, seed=N1).cuda()
    w2 = W.w_row_groups(N2, N1, 0.02, seed=N2 + 1).cuda()
    b1 = W.normal((N1,), 0.1, seed=3).cuda()
    b2 = W.normal((N2,), 0.1, seed=4).cuda()
    wq1, ws1 = fg8.quantize_weight(w1, fmt)
    wq2, ws2 = fg8.quantize_weight(w2, fmt)
    # reference: two independent layers
    y1_ref = fg8.linear(x, wq1, ws1, b1, fmt)
    y2_ref = fg8.linear(y1_ref, wq2, ws2, b2, fmt)
    # chained
    s = torch.cuda.current_stream().cuda_stream
    wsa, wsb = _ws(fg8, M, N1, K1, fmt), _ws(fg8, M, N2, N1, fmt)
    wsb.fill_(0xFF)  # stale bytes everywhere: the chain must write all it uses
    wsb[:256].zero_()
    y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
    y2 = torch.full((M, N2), float("nan"), dtype=torch.bfloat16, device="cuda")
    fg8.fg8_linear_prepare(x.data_ptr(), M, N1, K1, x.stride(0), ws1.data_ptr(), fmt, wsa.data_ptr(), wsa.numel(), s)
    fg8.fg8_linear_run_chain(wq1.data_ptr(), ws1.data_ptr(), b1.data_ptr(), y1.data_ptr(), M, N1, K1, N1, fmt,
                             wsa.data_ptr(), wsa.numel(), N2, ws2.data_ptr(), wsb.data_ptr(), wsb.numel(), s)
    fg8.fg8_linear_run(wq2.data_ptr(), ws2.data_ptr(), b2.data_ptr(), y2.data_ptr(), M, N2, N1, N2, fmt,
                       wsb.data_ptr(), wsb.numel(), s)
    torch.cuda.synchronize()
    assert torch.equal(y1, y1_ref)
    assert torch.equal(y2, y2_ref)
    assert fg8.fg8_check_device_status(wsa.data_ptr(), s) == 0
    assert fg8.fg8_check_device_status(wsb.data_ptr(), s) == 0



@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_linear_chain_three_layers(fg8, fmt):
    M, dims = 777, [384, 1024, 272, 512]
    x = W.x_student_t(M, dims[0], seed=11).cuda()
    layers, ref = [], x
    for i in range(3):
        w = W.w_row_groups(dims[i + 1], dims[i], 0.03, seed=20 + i).cuda()
        b = None if i == 1 else W.normal((dims[i + 1],), 0.1, seed=30 + i).cuda()
        wq, ws = fg8.quantize_weight(w, fmt)
        layers.append((wq, ws, b))
    ys = fg8.linear_chain(x, layers, fmt)
    torch.cuda.synchronize()
    for (wq, ws, b), y in zip(layers, ys):
        ref = fg8.linear(ref, wq, ws, b, fmt)
        assert torch.equal(y, ref)
