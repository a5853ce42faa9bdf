"""The shape rule that picks the few-token kernel (C++) and its mirror in
bench.py agree (the library's choice read back through fg8_linear_plan), and
the tiled GEMM's split-K tail plan behaves as documented."""
import pytest

import workloads as W


@pytest.fixture(scope="module")
def fg8():
    from fine_grained_fp8_act_b200 import build
    build.build()
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("M", [33, 64, 100, 128])
@pytest.mark.parametrize("N", [256, 1024, 4096, 9464, 9472, 9480, 12288, 14336])
def test_few_token_rule_matches_bench(fg8, M, N):
    import bench
    K = 8192
    lib_small = fg8.fg8_linear_plan(M, N, K, 0)[0] != 0
    bench_small = bench.layer_path(W.Gemm("t", M, K, N, 0)) != "tiled"
    assert lib_small == bench_small, (M, N, lib_small, bench_small)


def test_rule_boundaries(fg8):
    import bench
    g = lambda M, N, f=0: bench.layer_path(W.Gemm("t", M, 4096, N, f))
    assert g(32, 1 << 16) == "small" and g(33, 1 << 16) == "tiled"     # M <= 32: always few-token
    assert g(128, 9472) == "small" and g(128, 9480) == "tiled"           # ceil(N/256) <= 37
    assert g(129, 256) == "tiled"
    assert g(16, 4096, 1) == "fused" and g(17, 4096, 1) == "small" and g(16, 4096, 0) == "small"


@pytest.mark.parametrize("fmt", [0, 1])
def test_rule_through_the_plan(fg8, fmt):
    import bench
    for M, N in [(1, 4096), (16, 4096), (17, 4096), (32, 1 << 16), (33, 1 << 16), (128, 9472), (128, 9480)]:
        kind = fg8.fg8_linear_plan(M, N, 4096, fmt)[0]
        path = bench.layer_path(W.Gemm("t", M, 4096, N, fmt))
        assert kind == {"tiled": 0, "small": 1, "fused": 2}[path], (M, N, fmt, kind, path)


def test_split_tail_plan(fg8):
    """Whole waves on 148 SMs: no split.  Otherwise the last wave's tiles are
    split so that all their units fit one wave, where a unit's K-blocks plus
    the partials' write-back, wait and read-back beat a whole tile's K loop,
    with at least 64 K-blocks and two row blocks; after more than 6 whole
    waves only a split that saves over 60 K-block periods, after 16 none."""
    plan = fg8.fg8_linear_plan
    # 16384 x 12288 x 12288: 6144 tiles of 128 x 256, 76 in the last wave
    # (two units each would not fit one wave); 41 whole waves anyway
    assert plan(16384, 12288, 12288, 0) == (0, 256, 0, 1)
    # 2048 x 12288 x 12288: 768 tiles = 5 waves + 28; 5 units of 20 K-blocks
    assert plan(2048, 12288, 12288, 0) == (0, 256, 28, 5)
    assert plan(2048, 12288, 12288, 1) == (0, 256, 28, 5)
    # 512 tokens: 192 tiles = 1 wave + 44; 3 units of 32 K-blocks
    assert plan(512, 12288, 12288, 0) == (0, 256, 44, 3)
    # one row block (streams the weights), too few K-blocks, too many waves
    assert plan(64, 12288, 12288, 1) == (0, 128, 0, 1)
    assert plan(8176, 1920, 480, 0)[2:] == (0, 1)
    assert plan(4096, 14336, 4096, 0)[2:] == (0, 1)
    # 4096 x 12288 x 12288: 10 waves + 56 tiles; 2 units would save 41 periods
    assert plan(4096, 12288, 12288, 0)[2:] == (0, 1)
    # many waves, a nearly empty last wave, long K: 6 units of 24 K-blocks
    assert plan(8192, 7168, 18432, 1) == (0, 256, 16, 6)
    assert plan(6144, 7168, 18432, 0) == (0, 256, 12, 6)
    # 20480 x 4096: 2560 tiles = 17 whole waves + 44: never
    assert plan(20480, 4096, 18432, 0)[2:] == (0, 1)
    for M, N, K, fmt in [(4096, 4096, 14336, 0), (256, 2048, 8192, 0), (2560, 2048, 8192, 1), (2500, 2040, 8160, 0)]:
        kind, bn, tiles, s = plan(M, N, K, fmt)
        total = -(-M // 128) * -(-N // bn)
        assert kind == 0 and tiles == total % 148 and s >= 2 and tiles * s <= 148, (M, N, K, fmt)
