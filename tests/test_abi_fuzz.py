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


def test_block32_linear_host_checks(lib):
    rng = np.random.default_rng(3)
    for i in range(1200):
        M = _dim(rng, [0, 1, 200, 2048])
        N = _dim(rng, [8, 264, 4096])
        K = _dim(rng, [16, 32, 400])
        fmt = int(rng.choice([0, 1, 1, 3]))
        block = int(rng.choice([32, 32, 32, 64, 16]))
        ld_x = K + int(rng.choice([0, 0, 8, -8, 4]))
        ld_y = N + int(rng.choice([0, 0, 8, -8, 4]))
        x, wq, ws, y = (_ptr(rng, 16) for _ in range(4))
        bias = None if rng.random() < 0.3 else _ptr(rng, 16)
        shape_ok = block == 32 and fmt == 1 and 0 <= M <= MAXD and 0 < N <= MAXD and 0 < K <= MAXD
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
            if ld_x % 8 or ld_y % 8 or not all(_aligned(p, 16) for p in (x, wq, y) if p is not None) or \
                    (bias is not None and not _aligned(bias, 16)):
                broken.add(ALIGN)
            if not _aligned(wsp, 256) or nbytes < need:
                broken.add(WORKSPACE)
        got = lib.fg8_linear_block(x, M, N, K, ld_x, wq, ws, bias, y, ld_y, fmt, block, wsp, nbytes, None)
        _check(got, broken, M, f"fg8_linear_block case {i}: M={M} N={N} K={K} fmt={fmt} block={block}")
