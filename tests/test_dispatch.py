"""The shape rule that picks the few-token kernel (C++) and its mirror in
bench.py agree.  Without a GPU the library's choice shows in its workspace
size: with float scales the prepare layout does not depend on N, so extra
bytes are the few-token kernel's split-K partials (K = 8192 keeps the split
count above 1 wherever that kernel runs with at most 74 weight tiles)."""
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
    need = fg8.fg8_linear_workspace_bytes(M, N, K, 0)
    tiled_need = fg8.fg8_linear_workspace_bytes(M, 1 << 20, K, 0)  # far past the rule: tiled
    nt = -(-N // 128)
    lib_small = need > tiled_need
    bench_small = bench.layer_path(W.Gemm("t", M, K, N, 0)) != "tiled"
    if 148 // nt >= 2:  # the few-token kernel would split K: its choice is visible
        assert lib_small == bench_small, (M, N, lib_small, bench_small)
    else:  # one split, no partials either way; the rule itself says tiled here
        assert not lib_small and not bench_small


def test_rule_boundaries(fg8):
    import bench
    g = lambda M, N, f=0: bench.layer_path(W.Gemm("t", M, 4096, N, f))
    assert g(32, 1 << 16) == "small" and g(33, 1 << 16) == "tiled"     # M <= 32: always few-token
    assert g(128, 9472) == "small" and g(128, 9480) == "tiled"           # ceil(N/256) <= 37
    assert g(129, 256) == "tiled"
    assert g(16, 4096, 1) == "fused" and g(17, 4096, 1) == "small" and g(16, 4096, 0) == "small"
