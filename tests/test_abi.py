"""The C ABI without a GPU: libfg8.so loads, exports every function
include/fg8.h declares, and rejects bad arguments on the host before any
launch.  (No compute call runs here.)"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fg8.h")


@pytest.fixture(scope="module")
def fg8():
    from fine_grained_fp8_act_b200 import build
    build.build()
    import fine_grained_fp8_act_b200 as m
    m.lib()
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fg8_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fg8_quantize_weight", "fg8_quantize_act", "fg8_linear", "fg8_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(fg8):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", fg8.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    # the Python binding binds exactly the declared set
    assert sorted(fg8._capi.SIGNATURES) == names
    # nothing else leaks out of the library under an fg8_ name
    extra = [s for s in exported if s.startswith("fg8_") and s not in names]
    assert not extra, extra


def test_library_needs_no_driver_to_load(fg8):
    out = subprocess.run(["ldd", fg8.library_path()], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out  # the driver is resolved at call time only


def test_status_strings(fg8):
    for code in range(7):
        assert fg8.fg8_status_string(code) and "unknown" not in fg8.fg8_status_string(code)
    assert "unknown" in fg8.fg8_status_string(99)
    assert fg8.fg8_version() >= 100


L = None


def _raw(fg8):
    return fg8.lib()


FAKE = 0x10000  # a 16-byte-aligned non-null "device" address; never dereferenced on these paths


@pytest.mark.parametrize("args,expect", [
    # (M, N, K, ld_x, ld_y, fmt)
    ((16, 256, 256, 256, 256, 7), 1),      # bad format
    ((16, 256, 256, 256, 256, -1), 1),
    ((-1, 256, 256, 256, 256, 0), 1),      # negative M
    ((16, 0, 256, 256, 256, 0), 1),        # N = 0
    ((16, 256, 0, 256, 256, 0), 1),        # K = 0
    ((16, 256, 200, 200, 256, 0), 2),      # K % 16
    ((16, 252, 256, 256, 256, 0), 2),      # N % 8
    ((16, 256, 256, 255, 256, 0), 1),      # ld_x < K
    ((16, 256, 256, 256, 255, 0), 1),      # ld_y < N
    ((16, 256, 256, 260, 256, 0), 2),      # ld_x % 8
    ((1 << 31, 256, 256, 256, 256, 0), 1),  # M beyond int32
])
def test_linear_rejects_bad_shapes(fg8, args, expect):
    M, N, K, ldx, ldy, fmt = args
    st = _raw(fg8).fg8_linear(FAKE, M, N, K, ldx, FAKE, FAKE, None, FAKE, ldy, fmt, FAKE * 16, 1 << 40, None)
    assert st == expect


def test_linear_rejects_null_and_misaligned(fg8):
    raw = _raw(fg8)
    assert raw.fg8_linear(None, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, FAKE * 16, 1 << 40, None) == 1
    assert raw.fg8_linear(FAKE + 8, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, FAKE * 16, 1 << 40, None) == 2
    assert raw.fg8_linear(FAKE, 16, 256, 256, 256, FAKE, FAKE, FAKE + 2, FAKE, 256, 0, FAKE * 16, 1 << 40, None) == 2
    # workspace: null, misaligned, too small
    assert raw.fg8_linear(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, None, 1 << 40, None) == 4
    assert raw.fg8_linear(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, FAKE + 16, 1 << 40, None) == 4
    assert raw.fg8_linear(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, FAKE * 16, 100, None) == 4


def test_chain_rejects_bad_next_layer(fg8):
    raw = _raw(fg8)

    def chain(M, N, K, next_N, ws=FAKE * 16, next_ws=FAKE * 32):
        return raw.fg8_linear_run_chain(FAKE, FAKE, None, FAKE, M, N, K, N, 0, ws, 1 << 40, next_N, FAKE, next_ws,
                                        1 << 40, None)

    assert chain(16, 264, 256, 128) == 2      # the next layer's K (this N) must be a multiple of 16
    assert chain(16, 256, 256, 0) == 1        # next_N = 0
    assert chain(16, 256, 256, 252) == 2      # next_N % 8
    assert chain(16, 256, 256, 256, next_ws=None) == 4
    assert chain(0, 256, 256, 256) == 0       # empty batch
    assert raw.fg8_linear_run_chain(FAKE, FAKE, None, FAKE, 16, 256, 256, 256, 0, FAKE * 16, 1 << 40, 256, None,
                                    FAKE * 32, 1 << 40, None) == 1  # next layer's weight scales missing


def test_conversions_reject_bad_args(fg8):
    raw = _raw(fg8)
    assert raw.fg8_dequantize_weight(FAKE, 0, 256, FAKE, 0, FAKE, 256, None) == 1
    assert raw.fg8_dequantize_weight(FAKE, 256, 256, FAKE, 3, FAKE, 256, None) == 1
    assert raw.fg8_dequantize_weight(FAKE, 256, 256, FAKE, 0, FAKE, 255, None) == 1   # ld_w < K
    assert raw.fg8_dequantize_weight(FAKE, 256, 200, FAKE, 0, FAKE, 200, None) == 2   # K % 16
    assert raw.fg8_dequantize_weight(FAKE, 256, 256, FAKE, 0, FAKE, 260, None) == 2   # ld_w % 8
    assert raw.fg8_dequantize_weight(None, 256, 256, FAKE, 0, FAKE, 256, None) == 1
    assert raw.fg8_scale_to_ue8m0(FAKE, -1, FAKE, None, None) == 1
    assert raw.fg8_scale_to_ue8m0(None, 0, None, None, None) == 0          # empty: no-op
    assert raw.fg8_scale_to_ue8m0(FAKE + 2, 8, FAKE, None, None) == 2


def test_static_scheme_rejects_bad_args(fg8):
    raw = _raw(fg8)
    assert raw.fg8_quantize_act_static(FAKE, 4, 256, 256, None, FAKE, FAKE, None) == 1      # no scale
    assert raw.fg8_quantize_act_static(FAKE, 4, 200, 200, FAKE, FAKE, FAKE, None) == 2      # K % 16
    assert raw.fg8_quantize_act_static(FAKE, 4, 256, 256, FAKE + 2, FAKE, FAKE, None) == 2  # scale alignment
    assert raw.fg8_quantize_act_static(None, 0, 256, 256, None, None, None, None) == 0      # empty
    assert raw.fg8_linear_static(FAKE, 16, 256, 256, 256, None, FAKE, FAKE, None, FAKE, 256, FAKE * 16, 1 << 40,
                                 None) == 1
    assert raw.fg8_linear_static(FAKE, 16, 256, 256, 256, FAKE, FAKE, FAKE, None, FAKE, 256, None, 1 << 40,
                                 None) == 4


def test_empty_m_is_a_noop(fg8):
    raw = _raw(fg8)
    assert raw.fg8_linear(None, 0, 256, 256, 256, None, None, None, None, 256, 0, None, 0, None) == 0
    assert raw.fg8_quantize_act(None, 0, 256, 256, None, None, 0, None) == 0


def test_quantizers_reject_bad_args(fg8):
    raw = _raw(fg8)
    assert raw.fg8_quantize_act(FAKE, 4, 256, 256, FAKE, FAKE, 2, None) == 1
    assert raw.fg8_quantize_act(FAKE, 4, 120, 128, FAKE, FAKE, 0, None) == 2
    assert raw.fg8_quantize_act(FAKE, 4, 256, 128, FAKE, FAKE, 0, None) == 1
    assert raw.fg8_quantize_weight(FAKE, 0, 256, 256, FAKE, FAKE, 0, None) == 1
    assert raw.fg8_quantize_weight(FAKE, 256, 248, 248, FAKE, FAKE, 1, None) == 2
    assert raw.fg8_quantize_weight(None, 256, 256, 256, FAKE, FAKE, 1, None) == 1
    # one CTA per 128 x 128 block on a 2-D grid: at most 65535 row blocks
    assert raw.fg8_quantize_weight(FAKE, 65535 * 128 + 1, 256, 256, FAKE, FAKE, 0, None) == 1


def test_valid_call_without_gpu_reports_unsupported_device(fg8):
    """No CPU fallback: a well-formed call on a host without a B200 returns
    FG8_ERR_UNSUPPORTED_DEVICE instead of computing anything."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    raw = _raw(fg8)
    assert raw.fg8_quantize_act(FAKE, 4, 256, 256, FAKE, FAKE, 0, None) == 3


def test_workspace_sizes(fg8):
    f = fg8.fg8_linear_workspace_bytes
    assert f(16, 256, 256, 7) == 0
    assert f(16, 256, 200, 0) == 0
    a = f(8176, 1920, 480, 0)
    assert a >= 8176 * 480 + 4 * 8176 * 4
    b = f(8192, 18432, 7168, 1)
    assert b >= 8192 * 7168
    assert f(0, 256, 256, 0) > 0
    # few tokens with a long K: the swap-AB kernel's split-K partials come on
    # top (2 weight tiles, 64 K-blocks -> 32 splits, the 512 / M cap;
    # fp32 [tiles][splits][M][128])
    assert f(16, 256, 8192, 0) >= 32 * 16 * 256 * 4
    assert f(16, 256, 8192, 0) > f(16, 256, 128, 0) + 32 * 16 * 256 * 4 - 64 * 1024
    # pre-quantized GEMM: header + scales in the GEMM's layouts (x: K-major
    # float32 over 128-row-padded M; W: 16-byte entries per 128x128 block)
    assert fg8.fg8_gemm_workspace_bytes(16, 256, 256, 0) >= 256 + 2 * 128 * 4 + 2 * 2 * 16
    assert fg8.fg8_gemm_workspace_bytes(16, 256, 256, 1) >= 256 + 512 + 2 * 512


def test_split_tail_workspace(fg8):
    """The tiled GEMM's split-K tail: fg8_linear's workspace adds room for the
    fp32 partials of the last wave's split tiles (128 x 128 or 128 x 256 per
    unit, at most one wave of 148 units) on top of the layout that the
    expert-grouped layer (which never splits) shares with it, and nothing
    when both tile widths fill whole waves on 148 SMs."""
    raw = _raw(fg8)
    lin, grp = fg8.fg8_linear_workspace_bytes, raw.fg8_grouped_linear_workspace_bytes
    M = 148 * 128  # 148 tiles of 128 x 256, 296 of 128 x 128, for N = 256
    assert lin(M, 256, 4096, 0) == grp(M, 1, 256, 4096, 0)
    for M, N, K in [(256, 2048, 8192), (2560, 2048, 8192), (2048, 12288, 12288), (4096, 4096, 14336),
                    (8192, 7168, 18432)]:
        extra = lin(M, N, K, 0) - grp(M, 1, N, K, 0)
        assert extra > 0 and extra % (128 * 128 * 4) == 0 and extra <= 148 * 128 * 256 * 4 + 256, (M, N, K, extra)
        assert fg8.fg8_linear_fused_workspace_bytes(M, N, K, 0) > lin(M, N, K, 0)
    # too few K-blocks to pay for a split (the ESM-2 layer shapes), one row
    # block, many whole waves before a tail that a split would shorten too
    # little, or more than 16 whole waves
    for M, N, K in [(8176, 1920, 480), (64, 12288, 12288), (4096, 12288, 12288), (20480, 4096, 18432)]:
        assert lin(M, N, K, 0) == grp(M, 1, N, K, 0), (M, N, K)


def test_scale_fmt_validation(fg8):
    from fine_grained_fp8_act_b200 import scale_fmt_code
    assert scale_fmt_code("float") == 0 and scale_fmt_code("ue8m0") == 1
    for bad in ("Float", "e8m0", "fp32", 3, None):
        with pytest.raises(ValueError):
            scale_fmt_code(bad)


def test_grouped_rejects_bad_args(fg8):
    raw = _raw(fg8)
    big = 1 << 40
    args = lambda **kw: [kw.get(k, v) for k, v in (
        ("x", FAKE), ("M", 256), ("K", 256), ("ld_x", 256), ("re", FAKE), ("E", 4), ("N", 256), ("wq", FAKE),
        ("ws", FAKE), ("b", None), ("y", FAKE), ("ld_y", 256), ("fmt", 1), ("wsp", FAKE * 16), ("nb", big),
        ("s", None))]
    g = raw.fg8_grouped_linear
    assert g(*args(E=0)) == 1
    assert g(*args(E=70000)) == 1
    assert g(*args(E=1 << 20, N=4096)) == 1      # E * N past 2^31
    assert g(*args(fmt=2)) == 1
    assert g(*args(re=None)) == 1
    assert g(*args(K=200, ld_x=200)) == 2        # K % 16
    assert g(*args(N=260, ld_y=264)) == 2        # N % 8
    assert g(*args(re=FAKE + 2)) == 2            # int32 alignment
    assert g(*args(nb=1024)) == 4                # workspace too small
    assert g(*args(M=0, x=None, re=None, y=None)) == 0
    f = raw.fg8_grouped_linear_workspace_bytes
    # UE8M0: the weight scale-factor region holds every expert's 128-row tiles
    assert f(256, 8, 256, 1024, 1) > f(256, 1, 256, 1024, 1) + 7 * 2 * 2 * 512 - 256
    assert f(256, 8, 256, 1024, 0) == fg8.fg8_linear_workspace_bytes(256, 256, 1024, 0)
    assert f(256, 0, 256, 1024, 0) == 0


def test_block_size_rejects_bad_args(fg8):
    raw = _raw(fg8)
    assert raw.fg8_quantize_act_block(FAKE, 4, 256, 256, FAKE, FAKE, 0, 16, None) == 1       # block 16
    assert raw.fg8_quantize_act_block(FAKE, 4, 256, 256, FAKE, FAKE, 0, 96, None) == 1       # block 96
    assert raw.fg8_quantize_act_block(FAKE, 4, 120, 128, FAKE, FAKE, 1, 32, None) == 2      # K % 16
    assert raw.fg8_quantize_act_block(FAKE, 4, 120, 128, FAKE, FAKE, 0, 64, None) == 2
    assert raw.fg8_quantize_act_block(None, 0, 256, 256, None, None, 1, 32, None) == 0      # empty
    assert raw.fg8_quantize_weight_block(FAKE, 0, 256, 256, FAKE, FAKE, 1, 32, None) == 1
    assert raw.fg8_quantize_weight_block(FAKE, 256, 248, 248, FAKE, FAKE, 1, 32, None) == 2
    assert raw.fg8_quantize_weight_block(FAKE, 256, 256, 256, FAKE, FAKE, 0, 48, None) == 1
    for fmt in (0, 1):
        assert raw.fg8_linear_block_workspace_bytes(256, 256, 256, fmt, 16) == 0
        assert raw.fg8_linear_block_workspace_bytes(256, 256, 256, fmt, 128) == \
            raw.fg8_linear_workspace_bytes(256, 256, 256, fmt)
    # UE8M0: x codes + 2 x-scale chunks (K = 256: 2 K-blocks) + 2 row tiles x 2 W chunks, beyond the header
    for blk in (32, 64):
        assert raw.fg8_linear_block_workspace_bytes(256, 256, 256, 1, blk) >= 256 * 256 + 2 * 2 * 512 + 2 * 2 * 512
    # float: x codes + K-major float32 x scales [K / blk][256]
    assert raw.fg8_linear_block_workspace_bytes(256, 256, 256, 0, 32) >= 256 * 256 + 8 * 256 * 4
    assert raw.fg8_linear_block_workspace_bytes(256, 256, 256, 0, 64) >= 256 * 256 + 4 * 256 * 4
    lb = raw.fg8_linear_block
    assert lb(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, 16, FAKE * 16, 1 << 40, None) == 1
    assert lb(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 2, 32, FAKE * 16, 1 << 40, None) == 1
    assert lb(FAKE, 16, 256, 200, 200, FAKE, FAKE, None, FAKE, 256, 1, 32, FAKE * 16, 1 << 40, None) == 2
    assert lb(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 0, 64, None, 1 << 40, None) == 4
    assert lb(FAKE, 16, 256, 256, 256, FAKE, FAKE, None, FAKE, 256, 1, 32, None, 1 << 40, None) == 4


def test_batched_row_expert_rejects_bad_args(fg8):
    raw = _raw(fg8)
    f = raw.fg8_grouped_row_expert
    assert f(FAKE, 0, 256, FAKE, None) == 1
    assert f(FAKE, 4, -1, FAKE, None) == 1
    assert f(None, 4, 256, FAKE, None) == 1
    assert f(FAKE, 4, 100, FAKE, None) == 2       # slabs must be whole 128-row blocks
    assert f(FAKE + 2, 4, 256, FAKE, None) == 2
    assert f(None, 4, 0, None, None) == 0         # nothing to write
