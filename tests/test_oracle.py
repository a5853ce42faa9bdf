"""Pins for the CPU oracle: each check ties it to something other than itself.

- e4m3fn decode against PyTorch's float8_e4m3fn (a library routine) and the
  format's published extremes; encode against a brute-force nearest-code search
  and against PyTorch's round-to-nearest-even cast (after clamping to +-448).
- UE8M0 against the power-of-two invariants and PyTorch's float8_e8m0fnu decode.
- The quantizers against numpy float32 arithmetic and the brute-force encoder,
  element by element, with the scale-shape rule of [zh] §一.
- The GEMM against exact rational arithmetic (fractions.Fraction) on tiny and
  ragged inputs, plus closed-form special cases (x = 0, one-hot W, power-of-two
  scales where float and UE8M0 must agree).

[zh] = "Transformers 中的细粒度 FP8 量化：配置、DeepGEMM 加速路径与 UE8M0 缩放格式完全指南".
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

FLOAT, UE8M0 = 0, 1


# ----------------------------------------------------------- independent --
def torch_e4m3_table():
    """Value of every code 0..255 decoded by PyTorch (NaN codes included)."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def brute_encode(f32):
    """Nearest finite e4m3fn code by exhaustive search; ties to even mantissa;
    saturate at 448; keep the sign of the input (also for zero)."""
    table = torch_e4m3_table()
    codes = np.arange(0x7F)  # non-negative finite codes
    vals = table[codes]
    out = np.empty(f32.size, dtype=np.uint8)
    for i, f in enumerate(np.asarray(f32, dtype=np.float32).ravel()):
        a = abs(float(f))
        sign = 0x80 if math.copysign(1.0, float(f)) < 0 else 0
        if a >= 448.0:
            out[i] = sign | 0x7E
            continue
        d = np.abs(vals - a)
        best = d.min()
        cand = codes[d == best]
        if cand.size > 1:
            cand = cand[(cand & 1) == 0]
        out[i] = sign | int(cand[0])
    return out


def frac_bf16_rne(q: Fraction) -> int:
    """bf16 bits of the exact rational q rounded to nearest, ties to even."""
    if q == 0:
        return 0
    sign = 0x8000 if q < 0 else 0
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, -126) - 7)
    n = a / quantum
    lo = math.floor(n)
    rem = n - lo
    r = lo + 1 if (rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1)) else lo
    val = float(r * quantum)
    bits = int(np.array([val], dtype=np.float32).view(np.uint32)[0]) >> 16
    return sign | bits


def e8m0_value_exact(b):
    return Fraction(2) ** (int(b) - 127)


# ------------------------------------------------------------------ e4m3 --
def test_e4m3_decode_matches_torch(orc):
    t = torch_e4m3_table()
    for c in range(256):
        v = orc.e4m3_value(c)
        if (c & 0x7F) == 0x7F:
            assert math.isnan(v) and math.isnan(t[c])
        else:
            assert v == t[c], (c, v, t[c])


def test_e4m3_format_extremes(orc):
    finite = [orc.e4m3_value(c) for c in range(256) if (c & 0x7F) != 0x7F]
    assert len(finite) == 254
    assert max(finite) == 448.0 and orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9
    pos = [orc.e4m3_value(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(pos, pos[1:])), "codes 0x00..0x7E increase"


def test_e4m3_roundtrip_all_finite_codes(orc):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        v = orc.e4m3_value(c)
        back = orc.e4m3_encode(np.float32(v) if c != 0x80 else np.float32(-0.0))
        assert back == c, (hex(c), v, hex(back))


def test_e4m3_midpoints_tie_to_even(orc):
    for c in range(0x7E):
        lo, hi = orc.e4m3_value(c), orc.e4m3_value(c + 1)
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # exactly representable
        even = c if c % 2 == 0 else c + 1
        assert orc.e4m3_encode(mid) == even
        assert orc.e4m3_encode(-mid) == 0x80 | even
        below = np.nextafter(mid, np.float32(0))
        above = np.nextafter(mid, np.float32(1e9))
        assert orc.e4m3_encode(below) == c
        assert orc.e4m3_encode(above) == c + 1


def test_e4m3_saturation_and_sign(orc):
    for f in (448.0, float(np.nextafter(np.float32(448), np.float32(1e9))), 463.9, 464.0, 465.0, 1e30, float("inf")):
        assert orc.e4m3_encode(f) == 0x7E
        assert orc.e4m3_encode(-f) == 0xFE
    assert orc.e4m3_encode(0.0) == 0x00
    assert orc.e4m3_encode(-0.0) == 0x80
    assert orc.e4m3_encode(-1e-30) == 0x80
    assert orc.e4m3_encode(2.0 ** -10) == 0x00       # tie between 0 and 2^-9 -> even (0)
    assert orc.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 0x01


def test_e4m3_encode_brute_force_random(orc):
    rng = np.random.default_rng(1234)
    f = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * np.float32(30),
        (rng.standard_normal(1000) * 1e-3).astype(np.float32),
        rng.uniform(-470, 470, 1000).astype(np.float32),
    ])
    got = orc.e4m3_encode_many(f)
    want = brute_encode(f)
    assert np.array_equal(got, want)


def test_e4m3_encode_vs_torch_all_bf16_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    for scale in (1.0, 1.0 / 448.0, 0.37109375, 3.0e-3, 2.0 ** -126, 1234.5):
        with np.errstate(over="ignore"):
            q = (f / np.float32(scale)).astype(np.float32)
        q = q[np.isfinite(q)]
        got = orc.e4m3_encode_many(q)
        ref = torch.from_numpy(np.clip(q, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got, ref), scale


def test_bf16_rounding_brute_force(orc):
    """The output rounding, double -> bf16 round-to-nearest-even, against a
    brute-force search: the two bf16 neighbours of |v| among all finite bf16
    values (exact in double), the nearer one, the even mantissa on a tie.
    Random magnitudes over the whole range, bf16 subnormals, exact
    midpoints and their one-ulp neighbours, signed zeros."""
    bits = np.arange(0x0000, 0x7F80, dtype=np.uint32)                 # +0 ... largest finite
    vals = (bits << 16).view(np.float32).astype(np.float64)
    rng = np.random.default_rng(17)
    mids = (vals[:-1] + vals[1:]) / 2                                  # exact: 8-bit significands
    pick = rng.choice(mids.size, 400, replace=False)
    cases = list(mids[pick]) + list(np.nextafter(mids[pick], 0)) + list(np.nextafter(mids[pick], np.inf))
    cases += list(rng.uniform(-1, 1, 300) * np.exp2(rng.integers(-135, 127, 300)))
    cases += [0.0, -0.0, 1.0, -3.0, vals[-1], -vals[-1], 2.0 ** -133, 2.0 ** -134, 1.5 * 2.0 ** -134]
    for v in cases:
        a = abs(v)
        i = int(np.searchsorted(vals, a, side="right")) - 1            # vals[i] <= a < vals[i + 1]
        if vals[i] == a:
            b = i
        else:
            mid = (vals[i] + vals[i + 1]) / 2
            b = i if a < mid else i + 1 if a > mid else (i if i % 2 == 0 else i + 1)
        want = int(bits[b]) | (0x8000 if np.signbit(v) else 0)
        assert orc.bf16_from_double(float(v)) == want, (v, hex(want))


# ----------------------------------------------------------------- UE8M0 --
def test_e8m0_decode_matches_torch(orc):
    t = torch.arange(255, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    for b in range(1, 255):
        assert orc.e8m0_value(b) == t[b] == 2.0 ** (b - 127)


def test_e8m0_ceil_invariants(orc):
    rng = np.random.default_rng(7)
    s = np.concatenate([
        np.exp2(rng.uniform(-126, 126, 4000)).astype(np.float32),
        np.exp2(np.arange(-126, 127)).astype(np.float32),
        np.array([2.0 ** -126, 1.0, 448.0 / 448.0, 1.0 / 448.0, 3.0, 0.75, 2.0 ** 127 * 0.9], dtype=np.float32),
    ])
    for si in s:
        si = np.float32(si)
        if not (np.isfinite(si) and si >= np.float32(2.0 ** -126)):
            continue
        b = orc.e8m0_ceil_byte(si)
        assert 1 <= b <= 254
        p = e8m0_value_exact(b)
        exact = Fraction(float(si))
        assert p >= exact, (si, b)
        assert p < 2 * exact, (si, b)
        if math.frexp(float(si))[0] == 0.5:  # exact power of two maps to itself
            assert p == exact


# ---------------------------------------------------------- group scale --
def test_group_scale_rule(orc):
    assert orc.group_scale(448.0) == 1.0
    assert orc.group_scale(0.0) == 2.0 ** -126
    assert orc.group_scale(1e-40) == 2.0 ** -126
    rng = np.random.default_rng(3)
    for a in np.abs(rng.standard_normal(2000).astype(np.float32) * np.float32(50)):
        want = np.float32(a) / np.float32(448.0)  # numpy's IEEE float32 division
        want = max(want, np.float32(2.0 ** -126))
        assert np.float32(orc.group_scale(a)) == want


# ------------------------------------------------------ scale shape rule --
@pytest.mark.parametrize("N,K", [(1, 1), (127, 128), (128, 129), (129, 255), (255, 256), (480, 1920),
                                 (1920, 480), (1, 7168), (3, 12288), (129, 127), (256, 480)])
def test_scale_shape_rule(orc, N, K):
    """[zh] §一: weight_scale_inv has shape (ceil(out/128), ceil(in/128))."""
    rng = np.random.default_rng(N * 7 + K)
    w = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32)).to(torch.bfloat16)
    bits = w.view(torch.int16).numpy().view(np.uint16)
    for fmt in (FLOAT, UE8M0):
        wq, ws = orc.quantize_weight(bits, fmt)
        assert wq.shape == (N, K)
        assert ws.shape == (-(-N // 128), -(-K // 128))
        xq, xs = orc.quantize_act(bits, fmt)
        assert xs.shape == (N, -(-K // 128))


# -------------------------------------------------------- the quantizers --
def _bf16_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _check_group(orc, vals_f32, q_codes, scale_word, fmt):
    """One group: scale from its own amax, each code = brute-force RNE of x / s'."""
    amax = np.float32(np.max(np.abs(vals_f32))) if vals_f32.size else np.float32(0)
    s = max(np.float32(amax) / np.float32(448.0), np.float32(2.0 ** -126))
    if fmt == FLOAT:
        assert np.float32(scale_word) == s
        s_used = s
    else:
        b = int(scale_word)
        assert e8m0_value_exact(b) >= Fraction(float(s)) and e8m0_value_exact(b) < 2 * Fraction(float(s))
        s_used = np.float32(2.0 ** (b - 127))
    quot = (vals_f32 / s_used).astype(np.float32)
    assert np.array_equal(q_codes, brute_encode(quot))
    mags = np.abs(torch_e4m3_table()[q_codes])
    if fmt == FLOAT and amax > 0 and s > np.float32(2.0 ** -126):
        assert mags.max() == 448.0  # the group's largest magnitude lands on e4m3's largest
    assert mags.max() <= 448.0


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(3, 256), (2, 480), (1, 144), (4, 16), (2, 200)])
def test_quantize_act_groups(orc, fmt, M, K):
    g = torch.Generator().manual_seed(M * 1000 + K)
    x = torch.randn(M, K, generator=g) * 3
    x[0, : min(K, 40)] *= 50          # outliers in the first group
    if K > 128:
        x[-1, 128:256] = 0            # an all-zero group (or partial one)
    x = x.to(torch.bfloat16)
    xq, xs = orc.quantize_act(_bf16_bits(x), fmt)
    xf = x.float().numpy()
    Kb = -(-K // 128)
    for m in range(M):
        for gidx in range(Kb):
            k0, k1 = 128 * gidx, min(128 * gidx + 128, K)
            _check_group(orc, xf[m, k0:k1], xq[m, k0:k1], xs[m, gidx], fmt)


def test_quantize_act_zero_group_and_negative_zero(orc):
    x = torch.zeros(1, 256, dtype=torch.bfloat16)
    x[0, 5] = -0.0
    x[0, 130] = 1.0
    x[0, 131] = -0.0
    for fmt in (FLOAT, UE8M0):
        xq, xs = orc.quantize_act(_bf16_bits(x), fmt)
        if fmt == FLOAT:
            assert xs[0, 0] == np.float32(2.0 ** -126)
        else:
            assert xs[0, 0] == 1
        assert xq[0, 5] == 0x80 and xq[0, 0] == 0x00
        assert xq[0, 131] == 0x80


def test_quantize_act_ragged_tail_uses_real_elements(orc):
    """A 16-wide last group: its scale comes from those 16 channels alone."""
    x = torch.zeros(1, 144)
    x[0, :128] = 100.0
    x[0, 128:] = torch.linspace(-0.5, 0.25, 16)
    x = x.to(torch.bfloat16)
    xq, xs = orc.quantize_act(_bf16_bits(x), FLOAT)
    assert xs[0, 1] == np.float32(0.5) / np.float32(448)
    assert orc.e4m3_value(int(xq[0, 128])) == -448.0



def test_quantize_act_quotient_is_a_correctly_rounded_division(orc):
    """The element quotient is RN_f32(x / s), not x times a rounded reciprocal
    of s.  The two differ by at most one float32 ulp, which changes the e4m3
    code only when x / s sits on a rounding midpoint, so the group is built
    for that: its amax fixes a non-power-of-two scale s, and every other
    element is a bf16 value x with x / s exactly an e4m3 midpoint.  Expected
    codes: numpy's IEEE float32 division, then PyTorch's RNE cast."""
    codes = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (codes[:-1] + codes[1:]) / 2
    rows, separating = [], 0
    for amax in (0.765625, 1.53125, 0.8203125, 1.421875):
        s = np.float32(amax) / np.float32(448)
        xs = (mids * np.float64(s)).astype(np.float32)
        exact = (xs.astype(np.float64) == mids * np.float64(s)) & ((xs.view(np.uint32) & 0xFFFF) == 0) & (xs < amax)
        xs = xs[exact]
        assert 0 < xs.size < 128
        row = np.zeros(128, dtype=np.float32)
        row[0] = amax
        row[1:1 + xs.size] = xs
        row[64:64 + xs.size // 2] = -xs[: xs.size // 2]  # negative ones too
        rows.append(row)
        recip = (xs * (np.float32(1) / s)).astype(np.float32)
        e4 = lambda q: torch.from_numpy(np.ascontiguousarray(q)).to(torch.float8_e4m3fn).view(torch.uint8)
        separating += int((e4(recip) != e4(xs / s)).sum())
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    xq, xsc = orc.quantize_act(_bf16_bits(x), FLOAT)
    xf = x.float().numpy()
    want_q = (xf / xsc.astype(np.float32)).astype(np.float32)  # IEEE float32 division, row scale broadcast
    want = torch.from_numpy(want_q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(xq, want)
    assert separating >= 8  # cases on which a reciprocal-multiply quotient would round differently

@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("N,K", [(256, 256), (200, 144), (130, 480), (16, 32)])
def test_quantize_weight_blocks(orc, fmt, N, K):
    g = torch.Generator().manual_seed(N + 17 * K)
    w = torch.randn(N, K, generator=g) * 0.02
    Nb, Kb = -(-N // 128), -(-K // 128)
    for nb in range(Nb):  # very different magnitudes per block: a wrong block index shows
        for kb in range(Kb):
            w[128 * nb:128 * nb + 128, 128 * kb:128 * kb + 128] *= 2.0 ** (3 * nb - 2 * kb)
    w = w.to(torch.bfloat16)
    wq, ws = orc.quantize_weight(_bf16_bits(w), fmt)
    wf = w.float().numpy()
    for nb in range(Nb):
        for kb in range(Kb):
            blk = wf[128 * nb:min(128 * nb + 128, N), 128 * kb:min(128 * kb + 128, K)]
            q = wq[128 * nb:min(128 * nb + 128, N), 128 * kb:min(128 * kb + 128, K)]
            _check_group(orc, blk.ravel(), q.ravel(), ws[nb, kb], fmt)


# ---------------------------------------------------------------- GEMM --
def exact_linear(xq, xs, wq, ws, bias_bits, fmt, block=128):
    """y[m,n] = sum_k xhat*what + bias as exact rationals (PyTorch decode of codes)."""
    t = torch_e4m3_table()
    M, K = xq.shape
    N = wq.shape[0]

    def sc(v):
        return Fraction(float(np.float32(v))) if fmt == FLOAT else e8m0_value_exact(v)

    xh = [[Fraction(float(t[xq[m, k]])) * sc(xs[m, k // block]) for k in range(K)] for m in range(M)]
    wh = [[Fraction(float(t[wq[n, k]])) * sc(ws[n // block, k // block]) for k in range(K)] for n in range(N)]
    bias = None
    if bias_bits is not None:
        bias = (bias_bits.astype(np.uint32) << 16).view(np.float32)
    y = [[None] * N for _ in range(M)]
    bnd = [[None] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            prods = [xh[m][k] * wh[n][k] for k in range(K)]
            s = sum(prods, Fraction(0))
            if bias is not None:
                s += Fraction(float(bias[n]))
            y[m][n] = s
            bnd[m][n] = sum((abs(p) for p in prods), Fraction(0))
    return y, bnd


def _rand_operands(M, N, K, fmt, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g)).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if bias else None
    return _bf16_bits(x), _bf16_bits(w), (None if b is None else _bf16_bits(b))


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (2, 3, 130), (3, 17, 200), (2, 5, 256), (1, 130, 48), (3, 4, 7)])
def test_linear_vs_exact_rationals(orc, fmt, M, N, K):
    xb, wb, bb = _rand_operands(M, N, K, fmt, seed=M * 100 + N * 10 + K)
    xq, xs = orc.quantize_act(xb, fmt)
    wq, ws = orc.quantize_weight(wb, fmt)
    y64, bound, ybf = orc.linear_dequant(xq, xs, wq, ws, bb, fmt)
    ye, be = exact_linear(xq, xs, wq, ws, bb, fmt)
    gamma = K * 2.0 ** -52
    for m in range(M):
        for n in range(N):
            err = abs(Fraction(y64[m, n]) - ye[m][n])
            assert err <= Fraction(gamma) * be[m][n] + Fraction(1, 2 ** 1074), (m, n)
            assert abs(Fraction(bound[m, n]) - be[m][n]) <= Fraction(gamma) * be[m][n]
            assert ybf[m, n] == frac_bf16_rne(Fraction(y64[m, n]))


def test_linear_x_zero_gives_bias(orc):
    M, N, K = 4, 130, 144
    x = np.zeros((M, K), dtype=np.uint16)
    _, wb, bb = _rand_operands(M, N, K, FLOAT, seed=5)
    for fmt in (FLOAT, UE8M0):
        xq, xs = orc.quantize_act(x, fmt)
        wq, ws = orc.quantize_weight(wb, fmt)
        y64, bound, ybf = orc.linear_dequant(xq, xs, wq, ws, bb, fmt)
        assert np.all(bound == 0)
        assert np.array_equal(ybf, np.broadcast_to(bb, (M, N)))
        assert np.array_equal(y64, np.broadcast_to((bb.astype(np.uint32) << 16).view(np.float32).astype(np.float64), (M, N)))


def test_linear_one_hot_weights_select_columns(orc):
    """W[n, perm[n]] = c, else 0: y[m, n] = xhat[m, perm[n]] * what + bias[n] (catches
    transposed operands, wrong indices and sign errors)."""
    M, N, K = 3, 40, 272
    g = torch.Generator().manual_seed(11)
    perm = torch.randperm(K, generator=g)[:N]
    w = torch.zeros(N, K)
    w[torch.arange(N), perm] = -0.75
    x = (torch.randn(M, K, generator=g) * 4).to(torch.bfloat16)
    bias = (torch.randn(N, generator=g)).to(torch.bfloat16)
    for fmt in (FLOAT, UE8M0):
        xq, xs = orc.quantize_act(_bf16_bits(x), fmt)
        wq, ws = orc.quantize_weight(_bf16_bits(w.to(torch.bfloat16)), fmt)
        y64, _, _ = orc.linear_dequant(xq, xs, wq, ws, _bf16_bits(bias), fmt)
        t = torch_e4m3_table()
        for m in range(M):
            for n in range(N):
                k = int(perm[n])
                sx = float(xs[m, k // 128]) if fmt == FLOAT else 2.0 ** (int(xs[m, k // 128]) - 127)
                sw = float(ws[n // 128, k // 128]) if fmt == FLOAT else 2.0 ** (int(ws[n // 128, k // 128]) - 127)
                want = t[xq[m, k]] * sx * t[wq[n, k]] * sw + float(bias[n].float())
                assert y64[m, n] == want
                if fmt == UE8M0:   # 0.75/448 rounds up to 2^-9; 0.75 / 2^-9 = 384 is an e4m3 value
                    assert t[wq[n, k]] * sw == -0.75
                else:              # 448 * RN(0.75/448) is within one float32 ulp of 0.75
                    assert abs(t[wq[n, k]] * sw + 0.75) <= 0.75 * 2.0 ** -23


def test_linear_pow2_scales_float_equals_ue8m0(orc):
    """When every group/block amax is 448 * 2^j, the float scale is already a power
    of two, so both formats quantize identically and give the same y."""
    M, N, K = 4, 136, 256
    g = torch.Generator().manual_seed(21)
    t = torch_e4m3_table()
    finite = torch.from_numpy(t[:0x7F].copy())
    x = finite[torch.randint(0, 0x7F, (M, K), generator=g)] * torch.where(torch.rand(M, K, generator=g) < 0.5, -1.0, 1.0)
    w = finite[torch.randint(0, 0x7F, (N, K), generator=g)] * torch.where(torch.rand(N, K, generator=g) < 0.5, -1.0, 1.0)
    for m in range(M):
        for gi in range(2):
            x[m, 128 * gi] = 448.0
            x[m, 128 * gi:128 * gi + 128] *= 2.0 ** (m - gi)
    for nb in range(2):
        for kb in range(2):
            w[128 * nb, 128 * kb] = 448.0
            w[128 * nb:128 * nb + 128, 128 * kb:128 * kb + 128] *= 2.0 ** (-7 - nb + kb)
    xb, wb = _bf16_bits(x.to(torch.bfloat16)), _bf16_bits(w.to(torch.bfloat16))
    assert np.array_equal(x.to(torch.bfloat16).float().numpy(), x.numpy())  # exactly representable
    res = {}
    for fmt in (FLOAT, UE8M0):
        xq, xs = orc.quantize_act(xb, fmt)
        wq, ws = orc.quantize_weight(wb, fmt)
        res[fmt] = (xq, wq) + orc.linear_dequant(xq, xs, wq, ws, None, fmt)
    assert np.array_equal(res[FLOAT][0], res[UE8M0][0])
    assert np.array_equal(res[FLOAT][1], res[UE8M0][1])
    assert np.array_equal(res[FLOAT][2], res[UE8M0][2])
    # lossless quantization: y equals the exact product of the bf16 inputs
    exact = x.double() @ w.double().T
    assert np.array_equal(res[FLOAT][2], exact.numpy())


def test_linear_row_subset_matches_full(orc):
    M, N, K = 9, 24, 160
    xb, wb, bb = _rand_operands(M, N, K, FLOAT, seed=99)
    xq, xs = orc.quantize_act(xb, FLOAT)
    wq, ws = orc.quantize_weight(wb, FLOAT)
    full = orc.linear_dequant(xq, xs, wq, ws, bb, FLOAT)
    rows = np.array([8, 0, 3], dtype=np.int64)
    part = orc.linear_dequant(xq, xs, wq, ws, bb, FLOAT, rows=rows)
    for a, b in zip(full, part):
        assert np.array_equal(a[rows], b)


# ------------------------------------------- checkpoint conversions ([zh] §五, §七) --
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_dequantize_lossless_blocks(orc, fmt):
    """Blocks whose largest magnitude is 448 * 2^j and whose values are e4m3
    values times 2^j quantize losslessly (scale 2^j): Fp8Dequantize must give
    the original weights back, bit for bit."""
    N, K = 200, 272
    g = torch.Generator().manual_seed(31)
    finite = torch.from_numpy(torch_e4m3_table()[:0x7F].copy())
    w = finite[torch.randint(0, 0x7F, (N, K), generator=g)] * torch.where(torch.rand(N, K, generator=g) < 0.5, -1.0, 1.0)
    for nb in range(2):
        for kb in range(3):
            w[128 * nb, 128 * kb] = 448.0
            w[128 * nb:128 * nb + 128, 128 * kb:128 * kb + 128] *= 2.0 ** (-9 + 2 * nb - kb)
    wb = _bf16_bits(w.to(torch.bfloat16))
    assert np.array_equal(w.to(torch.bfloat16).double().numpy(), w.numpy())
    wq, ws = orc.quantize_weight(wb, fmt)
    assert np.array_equal(orc.dequantize_weight(wq, ws, fmt), wb)


def test_dequantize_vs_exact_rationals(orc):
    """Non-power-of-two float scales: every dequantized element is the exact
    rational value(q) * scale rounded once to bf16 (nearest, ties to even);
    decode by PyTorch's e4m3 table, products in fractions.Fraction."""
    N, K = 130, 144
    g = torch.Generator().manual_seed(32)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    wq, ws = orc.quantize_weight(_bf16_bits(w), FLOAT)
    out = orc.dequantize_weight(wq, ws, FLOAT)
    table = torch_e4m3_table()
    for n in range(0, N, 3):
        for k in range(0, K, 5):
            s = Fraction(float(ws[n // 128, k // 128]))
            want = frac_bf16_rne(Fraction(float(table[wq[n, k]])) * s)
            assert out[n, k] == want, (n, k)


def test_dequantize_within_half_step(orc):
    """|w - dequant(quant(w))| <= half an e4m3 step at the block's scale plus
    the bf16 rounding of the result."""
    N, K = 256, 384
    g = torch.Generator().manual_seed(33)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    for fmt in (FLOAT, UE8M0):
        wq, ws = orc.quantize_weight(_bf16_bits(w), fmt)
        back = torch.from_numpy(orc.dequantize_weight(wq, ws, fmt).astype(np.int16)).view(torch.bfloat16).double()
        s = torch.from_numpy(np.asarray(ws).astype(np.float64) if fmt == FLOAT else
                             np.ldexp(1.0, np.asarray(ws).astype(np.int64) - 127))
        s_full = s.repeat_interleave(128, 0)[:N].repeat_interleave(128, 1)[:, :K]
        a = (w.double() / s_full).abs()
        step = torch.where(a >= 2.0 ** -6, 2.0 ** (torch.floor(torch.log2(a.clamp(min=2.0 ** -6))) - 3), torch.full_like(a, 2.0 ** -9))
        bound = 0.5 * step * s_full + back.abs() * 2.0 ** -8
        assert bool(((w.double() - back).abs() <= bound).all())


def test_scale_to_e8m0_powers_of_two(orc):
    """s = 2^e, -127 <= e <= 127, converts to the UE8M0 byte e + 127, which
    PyTorch's float8_e8m0fnu decodes back to s."""
    e = np.arange(-127, 128)
    s = np.ldexp(np.float32(1.0), e).astype(np.float32)
    out, bad = orc.scale_to_e8m0(s)
    assert bad == 0
    assert np.array_equal(out.astype(np.int64), e + 127)
    back = torch.from_numpy(out.copy()).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(back, s.astype(np.float64))


def test_scale_to_e8m0_rejects_non_ue8m0_values(orc):
    """Values that are no UE8M0 scale (not a power of two, not positive,
    not finite, below 2^-127) become the UE8M0 NaN byte and are counted."""
    s = np.array([3.0, 1.5, 0.75 * 2.0 ** -100, 0.0, -0.0, -2.0, np.inf, -np.inf, np.nan, 2.0 ** -128, 2.0 ** -149,
                  np.float32(2.0 ** 127) * np.float32(1.0000001)], dtype=np.float32)
    out, bad = orc.scale_to_e8m0(s)
    assert bad == s.size
    assert (out == 255).all()


# ------------------------------------------------ static activation scheme --
def test_quantize_act_static_vs_brute_force(orc):
    """One float32 scale for the whole tensor: every code is the brute-force
    nearest e4m3 code of the numpy float32 quotient x / s (IEEE division),
    values beyond 448 s saturating."""
    M, K = 5, 272
    g = torch.Generator().manual_seed(41)
    x = (torch.randn(M, K, generator=g) * 3.0).to(torch.bfloat16)
    x[0, 0], x[1, 5], x[2, 7] = 3000.0, -5000.0, 0.0
    x[3, 9] = -0.0
    xb = _bf16_bits(x)
    for s in (np.float32(0.0123), np.float32(1.0), np.float32(2.0 ** -7), np.float32(3.7)):
        xq, xs = orc.quantize_act_static(xb, float(s))
        quot = x.float().numpy() / s
        assert np.array_equal(xq.ravel(), brute_encode(quot.ravel()))
        assert xs.shape == (M, 3) and (xs == s).all()


def test_quantize_act_static_lossless_and_linear(orc):
    """x = e4m3 value * 2^j with s = 2^j quantizes losslessly, and the linear
    layer on it equals the exact product (exact rationals)."""
    M, N, K = 3, 5, 144
    g = torch.Generator().manual_seed(42)
    finite = torch.from_numpy(torch_e4m3_table()[:0x7F].copy())
    codes = torch.randint(0, 0x7F, (M, K), generator=g)
    sign = torch.where(torch.rand(M, K, generator=g) < 0.5, -1.0, 1.0)
    x = finite[codes] * sign * 2.0 ** -3
    xb = _bf16_bits(x.to(torch.bfloat16))
    xq, xs = orc.quantize_act_static(xb, 2.0 ** -3)
    want = (codes.numpy().astype(np.uint8) | np.where(sign.numpy() < 0, 0x80, 0).astype(np.uint8))
    want[(codes.numpy() == 0) & (sign.numpy() < 0)] = 0x80
    assert np.array_equal(xq, want)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    wq, ws = orc.quantize_weight(_bf16_bits(w), FLOAT)
    y64, _, _ = orc.linear_dequant(xq, xs, wq, ws, None, FLOAT)
    table = torch_e4m3_table()
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(x[m, k])) * Fraction(float(table[wq[n, k]])) * Fraction(float(ws[n // 128, k // 128]))
                        for k in range(K))
            assert abs(Fraction(y64[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)


# ---------------------------------------------------------- MoE experts --
def _lossless_rows(M, K, rng, exps):
    """Rows whose 128-groups each have amax 448 * 2^i and every value on the
    e4m3 grid times 2^i: both scale formats then give s = 2^i exactly and
    quantization is lossless (all values are bf16 numbers)."""
    table = torch_e4m3_table()
    finite = table[np.isfinite(table)]
    x = np.empty((M, K))
    for m in range(M):
        for g in range(K // 128):
            i = exps[(m + g) % len(exps)]
            v = rng.choice(finite, 128) * 2.0 ** i
            v[rng.integers(128)] = 448.0 * 2.0 ** i * rng.choice([-1.0, 1.0])
            x[m, g * 128:(g + 1) * 128] = v
    return x


def _bits(a):
    return (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _moe_case(seed, fmt, E=3, K=256, M=4 * 128 + 50, tile_e=(2, 0, -1, 1, 0)):
    rng = np.random.default_rng(seed)
    N = K
    x = _lossless_rows(M, K, rng, (-12, -9, -6))
    perms = [rng.permutation(K) for _ in range(E)]
    c = [448.0 * 2.0 ** j for j in (-14, -10, -7)][:E]
    w = np.zeros((E, N, K))
    for e in range(E):
        w[e, np.arange(N), perms[e]] = c[e]   # W_e[n, pi_e(n)] = c_e
    b = _bits(rng.normal(0, 0.1, (E, N)))
    re = np.empty(M, dtype=np.int32)
    for t, e in enumerate(tile_e):
        re[t * 128:(t + 1) * 128] = e
    re[128 - 10:128] = -1  # padding rows inside a computed block: computed with the block's expert
    wq = np.empty((E, N, K), dtype=np.uint8)
    ws = np.empty((E, N // 128, K // 128), dtype=np.float32 if fmt == FLOAT else np.uint8)
    return x, perms, c, b, re, wq, ws, w


@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_grouped_linear_closed_form(orc, fmt):
    """Experts W_e = c_e * P_e (a permutation, c_e = 448 * 2^j, block scales
    exact) on losslessly quantized rows: y[r, n] = c_e * x[r, pi_e(n)] + b_e[n]
    exactly, with e the expert of r's 128-row block; skipped blocks untouched."""
    x, perms, c, b, re, wq, ws, w = _moe_case(7, fmt)
    for e in range(w.shape[0]):
        wq[e], ws[e] = orc.quantize_weight(_bits(w[e]), fmt)
    y64, bound, ybf, written = orc.grouped_linear(_bits(x), re, wq, ws, b, fmt)
    bf = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t, e in enumerate((2, 0, -1, 1, 0)):
        rows = np.arange(t * 128, min(x.shape[0], (t + 1) * 128))
        if e < 0:
            assert not written[rows].any() and np.isnan(y64[rows]).all()
            continue
        assert written[rows].all()
        want = c[e] * x[rows][:, perms[e]] + bf[e]
        assert np.array_equal(y64[rows], want), f"block {t} (expert {e})"


def test_grouped_linear_block_order(orc):
    """Moving whole 128-row blocks (rows and their expert) moves the outputs."""
    rng = np.random.default_rng(3)
    E, N, K, M = 3, 136, 384, 3 * 128 + 40
    x = _bits(rng.normal(0, 1, (M, K)))
    wq = np.empty((E, N, K), dtype=np.uint8)
    ws = np.empty((E, 2, 3), dtype=np.uint8)
    for e in range(E):
        wq[e], ws[e] = orc.quantize_weight(_bits(rng.normal(0, 0.05, (N, K))), UE8M0)
    re = np.repeat(np.array([1, 2, 0, 2], dtype=np.int32), 128)[:M]
    y1 = orc.grouped_linear(x, re, wq, ws, None, UE8M0)[0]
    order = [2, 0, 1]  # full blocks only; the ragged last block stays
    idx = np.concatenate([np.arange(o * 128, o * 128 + 128) for o in order] + [np.arange(384, M)])
    y2 = orc.grouped_linear(x[idx], re[idx], wq, ws, None, UE8M0)[0]
    assert np.array_equal(y2, y1[idx])


def test_grouped_linear_one_expert_is_the_dense_layer(orc):
    """One expert owning every block is the dense layer of [zh] §八 step 6."""
    rng = np.random.default_rng(4)
    M, N, K = 200, 264, 256
    x = _bits(rng.normal(0, 1, (M, K)))
    wq, ws = orc.quantize_weight(_bits(rng.normal(0, 0.05, (N, K))), FLOAT)
    b = _bits(rng.normal(0, 0.1, N))
    y64, bound, ybf, written = orc.grouped_linear(x, np.zeros(M, np.int32), wq[None], ws[None], b[None], FLOAT)
    d64, dbound, dbf = orc.linear(x, wq, ws, b, FLOAT)
    assert written.all() and np.array_equal(y64, d64) and np.array_equal(ybf, dbf)


def test_grouped_linear_rejects_unknown_expert(orc):
    x = np.zeros((128, 128), np.uint16)
    wq = np.zeros((2, 8, 128), np.uint8)
    ws = np.ones((2, 1, 1), np.float32)
    with pytest.raises(ValueError):
        orc.grouped_linear(x, np.full(128, 2, np.int32), wq, ws, None, FLOAT)



@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_grouped_linear_block_expert_is_its_first_row(orc, fmt):
    """Only row_expert[128 t] selects block t's expert (or skips it): the
    other rows of a block may hold anything, -1 and other experts included,
    and the whole block is still the dense layer of that one expert."""
    rng = np.random.default_rng(11)
    E, N, K, M = 3, 136, 256, 2 * 128 + 40
    x = _bits(rng.normal(0, 1, (M, K)))
    wq = np.empty((E, N, K), dtype=np.uint8)
    ws = np.empty((E, 2, 2), dtype=np.float32 if fmt == FLOAT else np.uint8)
    for e in range(E):
        wq[e], ws[e] = orc.quantize_weight(_bits(rng.normal(0, 0.05, (N, K))), fmt)
    b = _bits(rng.normal(0, 0.1, (E, N)))
    re = np.ones(M, dtype=np.int32)
    re[0], re[64], re[65], re[127] = 2, -1, 0, -1     # block 0: expert 2, whatever its other rows say
    re[128], re[129:256] = -1, 2                      # block 1: skipped
    re[256], re[257:] = 0, -1                         # block 2 (40 rows): expert 0
    y64, _, ybf, written = orc.grouped_linear(x, re, wq, ws, b, fmt)
    assert written[:128].all() and not written[128:256].any() and written[256:].all()
    for rows, e in ((np.arange(0, 128), 2), (np.arange(256, M), 0)):
        d64, _, dbf = orc.linear(x, wq[e], ws[e], b[e], fmt, rows=rows)
        assert np.array_equal(y64[rows], d64) and np.array_equal(ybf[rows], dbf)

# ------------------------------------- non-default block sizes 32 and 64 --
@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,K", [(3, 256), (2, 80), (1, 48), (2, 208)])
def test_quantize_act_groups_small_blocks(orc, fmt, M, K, blk):
    """1 x blk groups (weight_block_size = (blk, blk)): each group's scale from
    its own blk channels (a shorter last group from its real ones), codes by
    brute force."""
    g = torch.Generator().manual_seed(7 * M + K + blk)
    x = torch.randn(M, K, generator=g)
    for j in range(-(-K // blk)):  # very different magnitudes per group: a wrong group index shows
        x[:, blk * j:blk * j + blk] *= 2.0 ** (3 * (j % 5) - 6)
    x = x.to(torch.bfloat16)
    xq, xs = orc.quantize_act(_bf16_bits(x), fmt, blk)
    assert xs.shape == (M, -(-K // blk))
    xf = x.float().numpy()
    for m in range(M):
        for j in range(-(-K // blk)):
            k0, k1 = blk * j, min(blk * j + blk, K)
            _check_group(orc, xf[m, k0:k1], xq[m, k0:k1], xs[m, j], fmt)


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("N,K", [(64, 64), (40, 80), (96, 48), (136, 208)])
def test_quantize_weight_blocks_small_blocks(orc, fmt, N, K, blk):
    g = torch.Generator().manual_seed(N + 3 * K + blk)
    w = torch.randn(N, K, generator=g) * 0.02
    Nb, Kb = -(-N // blk), -(-K // blk)
    for nb in range(Nb):
        for kb in range(Kb):
            w[blk * nb:blk * nb + blk, blk * kb:blk * kb + blk] *= 2.0 ** (3 * nb - 2 * kb)
    w = w.to(torch.bfloat16)
    wq, ws = orc.quantize_weight(_bf16_bits(w), fmt, blk)
    assert ws.shape == (Nb, Kb)
    wf = w.float().numpy()
    for nb in range(Nb):
        for kb in range(Kb):
            blkv = wf[blk * nb:min(blk * nb + blk, N), blk * kb:min(blk * kb + blk, K)]
            q = wq[blk * nb:min(blk * nb + blk, N), blk * kb:min(blk * kb + blk, K)]
            _check_group(orc, blkv.ravel(), q.ravel(), ws[nb, kb], fmt)


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
@pytest.mark.parametrize("M,N,K", [(2, 3, 80), (1, 40, 64), (3, 5, 48), (2, 70, 144)])
def test_linear_vs_exact_rationals_small_blocks(orc, fmt, M, N, K, blk):
    g = torch.Generator().manual_seed(M * 31 + N * 7 + K + blk)
    x = torch.randn(M, K, generator=g)
    w = torch.randn(N, K, generator=g) * 0.02
    for j in range(-(-K // blk)):  # scales that differ by group, so a k / 128 index would show
        x[:, blk * j:blk * j + blk] *= 2.0 ** (2 * j - 3)
        w[:, blk * j:blk * j + blk] *= 2.0 ** (1 - j)
    for i in range(-(-N // blk)):  # and by row block, so a n / 128 index would show
        w[blk * i:blk * i + blk, :] *= 2.0 ** (3 - 2 * i)
    xb, wb = _bf16_bits(x.to(torch.bfloat16)), _bf16_bits(w.to(torch.bfloat16))
    bb = _bf16_bits((torch.randn(N, generator=g) * 0.1).to(torch.bfloat16))
    xq, xs = orc.quantize_act(xb, fmt, blk)
    wq, ws = orc.quantize_weight(wb, fmt, blk)
    y64, bound, ybf = orc.linear_dequant(xq, xs, wq, ws, bb, fmt, block=blk)
    ye, be = exact_linear(xq, xs, wq, ws, bb, fmt, block=blk)
    gamma = K * 2.0 ** -52
    for m in range(M):
        for n in range(N):
            assert abs(Fraction(y64[m, n]) - ye[m][n]) <= Fraction(gamma) * be[m][n] + Fraction(1, 2 ** 1074)
            assert ybf[m, n] == frac_bf16_rne(Fraction(y64[m, n]))
    y2 = orc.linear(xb, wq, ws, bb, fmt, block=blk)[0]
    assert np.array_equal(y2, y64)


@pytest.mark.parametrize("blk", [32, 64])
@pytest.mark.parametrize("fmt", [FLOAT, UE8M0])
def test_small_blocks_equal_block128_when_scales_coincide(orc, fmt, blk):
    """When every blk-group of a 128-group (and every blk x blk block of a
    128 x 128 block) has the same amax, the scales coincide and so do the
    codes and y: the smaller block reduces to the default layer."""
    rng = np.random.default_rng(9 + blk)
    M, N, K = 3, 136, 256
    x = rng.normal(0, 1, (M, K)).astype(np.float32)
    w = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    x = np.clip(x, -3.0, 3.0)
    x[:, ::blk] = 3.0                 # each blk-group holds the row's amax
    w = np.clip(w, -0.05, 0.05)
    for n0 in range(0, N, blk):       # each blk x blk block holds its 128 x 128 block's amax
        w[n0, ::blk] = 0.0625
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    wb = (w.view(np.uint32) >> 16).astype(np.uint16)
    b = (rng.normal(0, 0.1, N).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qs, ss = orc.quantize_weight(wb, fmt, blk)
    q128, s128 = orc.quantize_weight(wb, fmt)
    assert np.array_equal(qs, q128)
    ys = orc.linear(xb, qs, ss, b, fmt, block=blk)[0]
    y128 = orc.linear(xb, q128, s128, b, fmt)[0]
    assert np.array_equal(ys, y128)
