"""The layer inside CUDA graphs: a serving loop captures fg8_linear once and
replays it with new activations in the same buffers.  Each kernel path --
the tiled GEMM (with and without its split-K tail), the few-token kernel on
prepared activations and the one that quantizes x itself -- is captured on
its own stream after one eager call (which sets up the library's per-device
state), replayed with fresh inputs, and must give the eager call's bits with
a clean status word."""
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


@pytest.mark.parametrize("M,N,K,fmt", [(300, 520, 1040, FLOAT), (300, 520, 1040, UE8M0),  # tiled
                                       (256, 2048, 8192, FLOAT),                            # tiled, split-K tail
                                       (8, 1024, 2048, FLOAT),                               # few-token, prepared
                                       (8, 1024, 2048, UE8M0)])                              # few-token, fused
def test_graph_replay_matches_eager(fg8, M, N, K, fmt):
    w = W.w_row_groups(N, K, 0.02, seed=N + K).cuda()
    b = W.normal((N,), 0.1, seed=N).cuda()
    wq, ws = fg8.quantize_weight(w, fmt)
    x = W.x_outliers(M, K, seed=1).cuda()
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = fg8.fg8_linear_workspace_bytes(M, N, K, fmt)
    wsp = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()

    def call(stream):
        fg8.fg8_linear(x.data_ptr(), M, N, K, K, wq.data_ptr(), ws.data_ptr(), b.data_ptr(), y.data_ptr(), N, fmt,
                       wsp.data_ptr(), nb, stream)

    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(side.cuda_stream)  # eager, outside the capture
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        call(torch.cuda.current_stream().cuda_stream)
    for trial in range(3):
        x.copy_(W.x_outliers(M, K, seed=10 + trial).cuda())
        g.replay()
        torch.cuda.synchronize()
        got = y.clone()
        want = fg8.linear(x, wq, ws, b, fmt)
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"replay {trial} differs from the eager call"
    assert fg8.fg8_check_device_status(wsp.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    del g
