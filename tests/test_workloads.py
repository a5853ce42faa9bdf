"""The synthetic input recipe, on CPU: each generator draws what its
description says (distribution, outlier channels, per-128-row weight
magnitudes, clipping, seeds), once rounded to bf16."""
import torch

import workloads as W


def _is_bf16_of_fp32(t):
    return t.dtype == torch.bfloat16 and torch.equal(t, t.float().to(torch.bfloat16))


def test_normal_is_seeded_and_scaled():
    a, b, c = W.normal((256, 512), 0.02, seed=7), W.normal((256, 512), 0.02, seed=7), W.normal((256, 512), 0.02, 8)
    assert _is_bf16_of_fp32(a) and torch.equal(a, b) and not torch.equal(a, c)
    std = a.float().std().item()
    assert abs(std / 0.02 - 1) < 0.02 and abs(a.float().mean().item()) < 0.02 * 0.02


def test_outlier_channels():
    """round(0.01 K) channels of N(0, 1) scaled by 20, the same channels in every row."""
    M, K = 256, 4096
    x = W.x_outliers(M, K, seed=3).float()
    col_std = x.std(dim=0)
    big = (col_std > 8).nonzero().flatten()
    assert big.numel() == round(0.01 * K)
    assert torch.all((col_std[big] > 15) & (col_std[big] < 25))
    rest = torch.ones(K, dtype=torch.bool)
    rest[big] = False
    assert abs(col_std[rest].mean().item() - 1) < 0.05 and col_std[rest].max().item() < 1.5


def test_student_t_clipped():
    """Student-t with 4 degrees of freedom clipped to +-50: variance near nu / (nu - 2) = 2, heavy tails."""
    x = W.x_student_t(512, 1024, seed=4).float()
    assert x.abs().max().item() <= 50.0
    var = x.var().item()
    assert 1.7 < var < 2.3
    z = (x - x.mean()) / x.std()
    assert (z ** 4).mean().item() > 4.0  # a normal's kurtosis is 3


def test_weight_row_group_magnitudes():
    """W ~ N(0, std^2) times one factor g = exp(U(ln 1/4, ln 4)) per 128-row group."""
    N, K, std = 1024 + 64, 2048, 0.015
    w = W.w_row_groups(N, K, std, seed=9).float()
    groups = -(-N // 128)
    g = torch.tensor([w[128 * i: 128 * i + 128].std().item() / std for i in range(groups)])
    assert torch.all((g > 0.25 * 0.97) & (g < 4.0 * 1.03))
    assert g.max() / g.min() > 1.5  # the groups differ
    for i in range(groups):  # one factor per group: every row of a group has about the same spread
        rows = w[128 * i: min(128 * i + 128, N)].std(dim=1) / std
        assert (rows.max() / rows.min()).item() < 1.3, i
    assert _is_bf16_of_fp32(W.w_row_groups(N, K, std, seed=9))


def test_config_seeds_and_shapes():
    """Config i draws from base seed i - 1: x at +0, W1 at +1, W2 at +2, bias at +3 (+10 for stage 2)."""
    x, w, b = W.make_inputs("tiny", W.TINY)
    assert (x.shape, w.shape, b.shape) == ((16, 256), (256, 256), (256,))
    assert torch.equal(x, W.x_normal(16, 256, 0)) and torch.equal(w, W.normal((256, 256), 0.02, 1))
    assert torch.equal(b, W.normal((256,), 0.1, 3))
    x1, w1, b1 = W.make_inputs("esm2", W.ESM_W1, stage=1)
    x2, w2, b2 = W.make_inputs("esm2", W.ESM_W2, stage=2)
    assert x1.shape == (8176, 480) and w1.shape == (1920, 480) and w2.shape == (480, 1920)
    assert torch.equal(w2, W.normal((480, 1920), 0.02, 1 + 2)) and torch.equal(b2, W.normal((480,), 0.1, 1 + 13))
    g = W.llama(16, "down")
    x, w, _ = W.make_inputs("llama", g, stage=2)
    assert (g.M, g.K, g.N) == (16, 14336, 4096) and torch.equal(x, W.x_outliers(16, 14336, 2))
    assert W.DSV3_UP.fmt == W.FMT_UE8M0 and W.square(64, 0).fmt == W.FMT_FLOAT
    x, w, _ = W.make_inputs("dsv3", W.Gemm("t", 4, 256, 384, 1))
    assert torch.equal(x, W.x_student_t(4, 256, 3)) and torch.equal(w, W.w_row_groups(384, 256, 0.015, 3 + 1))
