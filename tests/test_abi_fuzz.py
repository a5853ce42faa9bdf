"""Seeded fuzzing of the C ABI's host-side checks (no GPU needed).

Every argument set that breaks one of the rules include/fg8.h documents must
come back with that rule's status before anything reaches the device: a
shape, format or leading-dimension problem (FG8_ERR_INVALID_ARG), an
alignment problem (FG8_ERR_ALIGNMENT) or a missing, misaligned or short
workspace (FG8_ERR_WORKSPACE).  Argument sets that break none return FG8_OK
for M = 0 and otherwise FG8_ERR_UNSUPPORTED_DEVICE, since this host has no
B200: the call got as far as looking for the device.  Where several rules
are broken, any of their statuses is accepted (the header fixes no order).
Pointers are never dereferenced on these paths.
"""
import numpy as np
import pytest

OK, INVALID, ALIGN, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3, 4
MAXD = 2**31 - 1
BASE = 1 << 24            # a 256-byte aligned address that is never dereferenced


@pytest.fixture(scope="module")
def lib():
    import torch
    if torch.cuda.is_available():
        pytest.skip("with a GPU present, well-formed calls would launch")
    import fine_grained_fp8_act_b200 as fg8
    return fg8.lib()


def _ptr(rng, align):
    """An address: usually aligned to `align`, sometimes off by 8 or 4, sometimes NULL."""
    r = rng.random()
    if r < 0.06:
        return None
    if r < 0.14:
        return BASE + 8
    if r < 0.18:
        return BASE + 4
    return BASE + (align if rng.random() < 0.5 else 0)


def _dim(rng, good):
    r = rng.random()
    if r < 0.05:
        return int(rng.choice([0, -1, MAXD + 1, 2**40]))
    if r < 0.15:
        return int(rng.choice(good)) + int(rng.choice([1, 4, 8]))
    return int(rng.choice(good))


def _aligned(p, a):
    return p is not None and p % a == 0


def _check(got, broken, M, what):
    if broken:
        assert got in broken, f"{what}: status {got}, expected one of {sorted(broken)}"
    else:
        assert got == (OK if M == 0 else UNSUPPORTED), f"{what}: status {got} for a well-formed call"


def test_linear_host_checks(lib):
    rng = np.random.default_rng(1)
    for i in range(1500):
        M = _dim(rng, [0, 1, 5, 16, 40, 300, 8192])
        N = _dim(rng, [8, 16, 264, 4096])
        K = _dim(rng, [16, 32, 400, 7168])
        fmt = int(rng.choice([0, 1, 1, 2]))
        ld_x = K + int(rng.choice([0, 0, 8, -8, 4]))
        ld_y = N + int(rng.choice([0, 0, 8, -8, 4]))
        x, wq, ws, y = (_ptr(rng, 16) for _ in range(4))
        bias = None if rng.random() < 0.3 else _ptr(rng, 16)
        shape_ok = fmt in (0, 1) and 0 <= M <= MAXD and 0 < N <= MAXD and 0 < K <= MAXD
        need = lib.fg8_linear_workspace_bytes(M, N, K, fmt) if shape_ok and K % 16 == 0 and N % 8 == 0 else 0
        wsp = _ptr(rng, 256)
        nbytes = int(rng.choice([need, need, need + 4096, max(need - 1, 0), 0]))
        broken = set()
        if not shape_ok or ld_x < K or ld_y < N:
            broken.add(INVALID)
        if shape_ok and (K % 16 or N % 8):
            broken.add(ALIGN)
        if shape_ok and M > 0:
            if None in (x, wq, ws, y):
                broken.add(INVALID)
            if ld_x % 8 or ld_y % 8 or not all(_aligned(p, 16) for p in (x, wq, ws, y) if p is not None) or \
                    (bias is not None and not _aligned(bias, 16)):
                broken.add(ALIGN)
            if not _aligned(wsp, 256) or nbytes < need:
                broken.add(WORKSPACE)
        got = lib.fg8_linear(x, M, N, K, ld_x, wq, ws, bias, y, ld_y, fmt, wsp, nbytes, None)
        _check(got, broken, M, f"fg8_linear case {i}: M={M} N={N} K={K} fmt={fmt} ld={ld_x},{ld_y}")


def test_grouped_linear_host_checks(lib):
    rng = np.random.default_rng(2)
    for i in range(1200):
        M = _dim(rng, [0, 128, 300, 4096])
        N = _dim(rng, [8, 264, 2048])
        K = _dim(rng, [16, 400, 7168])
        E = int(rng.choice([1, 3, 256, 0, 70000]))
        fmt = int(rng.choice([0, 1, 1, 5]))
        ld_x = K + int(rng.choice([0, 0, 8, -8, 4]))
        ld_y = N + int(rng.choice([0, 0, 8, -8, 4]))
        x, wq, ws, y = (_ptr(rng, 16) for _ in range(4))
        re = None if rng.random() < 0.05 else BASE + int(rng.choice([0, 0, 4, 2]))
        bias = None if rng.random() < 0.3 else _ptr(rng, 16)
        shape_ok = fmt in (0, 1) and 0 <= M <= MAXD and 0 < N <= MAXD and 0 < K <= MAXD
        groups_ok = shape_ok and 0 < E <= 65535 and E * N + 256 <= MAXD and \
            E * -(-N // 128) * -(-K // 128) <= MAXD
        need = (lib.fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt)
                if groups_ok and K % 16 == 0 and N % 8 == 0 else 0)
        wsp = _ptr(rng, 256)
        nbytes = int(rng.choice([need, need, max(need - 1, 0), 0]))
        broken = set()
        if not groups_ok or ld_x < K or ld_y < N:
            broken.add(INVALID)
        if shape_ok and (K % 16 or N % 8):
            broken.add(ALIGN)
        if groups_ok and M > 0:
            if None in (x, wq, ws, y, re):
                broken.add(INVALID)
            if ld_x % 8 or ld_y % 8 or not all(_aligned(p, 16) for p in (x, wq, ws, y) if p is not None) or \
                    (bias is not None and not _aligned(bias, 16)) or (re is not None and re % 4):
                broken.add(ALIGN)
            if not _aligned(wsp, 256) or nbytes < need:
                broken.add(WORKSPACE)
        got = lib.fg8_grouped_linear(x, M, K, ld_x, re, E, N, wq, ws, bias, y, ld_y, fmt, wsp, nbytes, None)
        _check(got, broken, M, f"fg8_grouped_linear case {i}: M={M} E={E} N={N} K={K} fmt={fmt}")


def test_small_block_linear_host_checks(lib):
    """fg8_linear_block at blocks 32 and 64 (both scale formats; other block
    sizes and formats refused)."""
    rng = np.random.default_rng(3)
    for i in range(1600):
        M = _dim(rng, [0, 1, 200, 2048])
        N = _dim(rng, [8, 264, 4096])
        K = _dim(rng, [16, 32, 400])
        fmt = int(rng.choice([0, 1, 1, 3]))
        block = int(rng.choice([32, 32, 64, 64, 16]))
        ld_x = K + int(rng.choice([0, 0, 8, -8, 4]))
        ld_y = N + int(rng.choice([0, 0, 8, -8, 4]))
        x, wq, ws, y = (_ptr(rng, 16) for _ in range(4))
        bias = None if rng.random() < 0.3 else _ptr(rng, 16)
        shape_ok = block in (32, 64) and fmt in (0, 1) and 0 <= M <= MAXD and 0 < N <= MAXD and 0 < K <= MAXD
        need = (lib.fg8_linear_block_workspace_bytes(M, N, K, fmt, block)
                if shape_ok and K % 16 == 0 and N % 8 == 0 else 0)
        wsp = _ptr(rng, 256)
        nbytes = int(rng.choice([need, need, max(need - 1, 0), 0]))
        broken = set()
        if not shape_ok or ld_x < K or ld_y < N:
            broken.add(INVALID)
        if shape_ok and (K % 16 or N % 8):
            broken.add(ALIGN)
        if shape_ok and M > 0:
            if None in (x, wq, ws, y):
                broken.add(INVALID)
            if ld_x % 8 or ld_y % 8 or not all(_aligned(p, 16) for p in (x, wq, ws, y) if p is not None) or \
                    (bias is not None and not _aligned(bias, 16)):
                broken.add(ALIGN)
            if not _aligned(wsp, 256) or nbytes < need:
                broken.add(WORKSPACE)
        got = lib.fg8_linear_block(x, M, N, K, ld_x, wq, ws, bias, y, ld_y, fmt, block, wsp, nbytes, None)
        _check(got, broken, M, f"fg8_linear_block case {i}: M={M} N={N} K={K} fmt={fmt} block={block}")


def _check_allowed(got, allowed, what):
    assert got in allowed, f"{what}: status {got}, expected one of {sorted(allowed)}"


@pytest.mark.parametrize("block", [None, 128, 32, 64])
def test_quantize_act_host_checks(lib, block):
    """fg8_quantize_act (block None) and fg8_quantize_act_block."""
    rng = np.random.default_rng(4 + (block or 0))
    for i in range(800):
        M = _dim(rng, [0, 1, 129, 8192])
        K = _dim(rng, [16, 48, 400, 7168])
        fmt = int(rng.choice([0, 1, 1, 2]))
        ld_x = K + int(rng.choice([0, 0, 8, -8, 4]))
        x, xq, xs = (_ptr(rng, 16) for _ in range(3))
        invalid = fmt not in (0, 1) or not (0 <= M <= MAXD and 0 < K <= MAXD) or ld_x < K or \
            block not in (None, 128, 64, 32)
        if invalid:
            allowed = {INVALID}
        elif M == 0:
            allowed = {OK}
        else:
            broken = set()
            if None in (x, xq, xs):
                broken.add(INVALID)
            if K % 16 or ld_x % 8 or not all(_aligned(p, 16) for p in (x, xq) if p is not None):
                broken.add(ALIGN)
            allowed = broken or {UNSUPPORTED}
        if block is None:
            got = lib.fg8_quantize_act(x, M, K, ld_x, xq, xs, fmt, None)
        else:
            got = lib.fg8_quantize_act_block(x, M, K, ld_x, xq, xs, fmt, block, None)
        _check_allowed(got, allowed, f"quantize_act block={block} case {i}: M={M} K={K} fmt={fmt} ld={ld_x}")


@pytest.mark.parametrize("block", [None, 128, 64, 32, 16])
def test_quantize_weight_host_checks(lib, block):
    """fg8_quantize_weight (block None) and fg8_quantize_weight_block."""
    rng = np.random.default_rng(40 + (block or 0))
    for i in range(800):
        N = int(rng.choice([65535 * 128, 65535 * 128 + 1])) if rng.random() < 0.05 else _dim(rng, [1, 264, 4096])
        K = _dim(rng, [16, 48, 400, 7168])
        fmt = int(rng.choice([0, 1, 1, 2]))
        ld_w = K + int(rng.choice([0, 0, 8, -8, 4]))
        w, wq, ws = (_ptr(rng, 16) for _ in range(3))
        b = 128 if block is None else block
        invalid = fmt not in (0, 1) or not (0 < N <= MAXD and 0 < K <= MAXD) or ld_w < K or \
            b not in (128, 64, 32) or None in (w, wq, ws)
        if not invalid and b == 128 and -(-N // 128) > 65535:
            invalid = True
        if not invalid and b in (32, 64) and -(-N // b) * -(-K // b) > MAXD // 8:
            invalid = True
        align = not invalid and (K % 16 or ld_w % 8 or not (_aligned(w, 16) and _aligned(wq, 16)))
        allowed = ({INVALID} | ({ALIGN} if (K % 16 or ld_w % 8) else set())) if invalid else \
            ({ALIGN} if align else {UNSUPPORTED})
        if block is None:
            got = lib.fg8_quantize_weight(w, N, K, ld_w, wq, ws, fmt, None)
        else:
            got = lib.fg8_quantize_weight_block(w, N, K, ld_w, wq, ws, fmt, block, None)
        _check_allowed(got, allowed, f"quantize_weight block={block} case {i}: N={N} K={K} fmt={fmt} ld={ld_w}")


def test_dequantize_and_scale_conversion_host_checks(lib):
    rng = np.random.default_rng(9)
    for i in range(800):
        N = _dim(rng, [1, 300, 4096])
        K = _dim(rng, [16, 400, 7168])
        fmt = int(rng.choice([0, 1, 1, 7]))
        ld_w = K + int(rng.choice([0, 0, 8, -8, 4]))
        wq, ws, w = (_ptr(rng, 16) for _ in range(3))
        invalid = fmt not in (0, 1) or not (0 < N <= MAXD and 0 < K <= MAXD) or ld_w < K or N * K > 2**40 or \
            None in (wq, ws, w)
        align = K % 16 or ld_w % 8 or not (_aligned(wq, 16) and _aligned(w, 16))
        allowed = ({INVALID} | ({ALIGN} if (K % 16 or ld_w % 8) else set())) if invalid else \
            ({ALIGN} if align else {UNSUPPORTED})
        got = lib.fg8_dequantize_weight(wq, N, K, ws, fmt, w, ld_w, None)
        _check_allowed(got, allowed, f"dequantize_weight case {i}: N={N} K={K} fmt={fmt} ld={ld_w}")

        n = int(rng.choice([-1, 0, 1, 1000, 2**20]))
        s, out = _ptr(rng, 4), _ptr(rng, 1)
        cnt = None if rng.random() < 0.3 else BASE + int(rng.choice([0, 0, 4, 2]))
        if n < 0:
            allowed = {INVALID}
        elif n == 0:
            allowed = {OK}
        else:
            broken = set()
            if s is None or out is None:
                broken.add(INVALID)
            if (s is not None and s % 4) or (cnt is not None and cnt % 4):
                broken.add(ALIGN)
            allowed = broken or {UNSUPPORTED}
        got = lib.fg8_scale_to_ue8m0(s, n, out, cnt, None)
        _check_allowed(got, allowed, f"scale_to_ue8m0 case {i}: n={n}")


def test_batched_row_expert_host_checks(lib):
    rng = np.random.default_rng(12)
    for i in range(800):
        E = int(rng.choice([1, 8, 256, 65535, 65536, 0, -3]))
        cap = int(rng.choice([0, 128, 256, 640, 100, -128, 2**31]))
        counts = None if rng.random() < 0.06 else BASE + int(rng.choice([0, 0, 2]))
        re = None if rng.random() < 0.06 else BASE + int(rng.choice([0, 0, 2]))
        if not (0 < E <= 65535) or cap < 0 or E * cap > MAXD:
            allowed = {INVALID}
        elif cap == 0:
            allowed = {OK}
        elif counts is None or re is None:
            allowed = {INVALID} | ({ALIGN} if cap % 128 else set())
        else:
            align = cap % 128 or counts % 4 or re % 4
            allowed = {ALIGN} if align else {UNSUPPORTED}
        got = lib.fg8_grouped_row_expert(counts, E, cap, re, None)
        _check_allowed(got, allowed, f"grouped_row_expert case {i}: E={E} cap={cap}")
