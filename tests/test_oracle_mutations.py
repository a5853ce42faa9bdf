"""The oracle's pins catch planted mistakes (CPU only; test infrastructure).

Each case copies the oracle with one plausible mistake planted in it: a
rounding or tie rule, a constant, a dropped term or element, a wrong or
transposed index, a lost sign (in the C++ source), or a wrong tile, expert,
bias or skip rule (in the Python grouped layer).  A C++ copy is compiled into
a temporary directory; a Python copy runs from a temporary copy of the tree.
The oracle's pin tests (tests/test_oracle.py) then run against it in a child
process, and at least one pin must fail.  An unmodified copy, built the same
way, must pass them all (the control).  Every planted mistake keeps each
memory access inside its buffer.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fg8_oracle.cpp")

# name: (text in the source, planted replacement)
MUTATIONS = {
    "e4m3 ties away from even": ("pick = (lo & 1) == 0 ? lo : hi;", "pick = hi;"),
    "e4m3 saturates to NaN": ("if (a >= kE4m3Max) return sign | 0x7E;", "if (a >= kE4m3Max) return sign | 0x7F;"),
    "e4m3 drops the sign of zero": ("const uint8_t sign = std::signbit(f) ? 0x80 : 0x00;",
                                    "const uint8_t sign = f < 0.0f ? 0x80 : 0x00;"),
    "UE8M0 rounds down": ("return static_cast<uint8_t>(mant == 0 ? biased : biased + 1);",
                          "return static_cast<uint8_t>(biased);"),
    "UE8M0 moves exact powers up": ("return static_cast<uint8_t>(mant == 0 ? biased : biased + 1);",
                                    "return static_cast<uint8_t>(biased + 1);"),
    "scale constant 440": ("float s = amax / 448.0f;", "float s = amax / 440.0f;"),
    "scale floor dropped": ("if (s < floor_s) s = floor_s;", "(void)floor_s;"),
    "quotient by reciprocal": ("const float quotient = bf16_to_float(x[m * ld_x + k]) / s_used;",
                               "const float quotient = bf16_to_float(x[m * ld_x + k]) * (1.0f / s_used);"),
    "act amax skips a group's last element": (
        "for (int64_t k = k0; k < k1; ++k) amax = std::fmax(amax, std::fabs(bf16_to_float(x[m * ld_x + k])));",
        "for (int64_t k = k0; k < k1 - 1; ++k) amax = std::fmax(amax, std::fabs(bf16_to_float(x[m * ld_x + k])));"),
    "weight amax skips a block's last row": (
        "for (int64_t n = n0; n < n1; ++n)\n        for (int64_t k = k0; k < k1; ++k) amax",
        "for (int64_t n = n0; n < n1 - 1; ++n)\n        for (int64_t k = k0; k < k1; ++k) amax"),
    "weight scales stored transposed": ("static_cast<float*>(w_scale_inv)[nb * Kb + kb] = s;",
                                        "static_cast<float*>(w_scale_inv)[kb * Nb + nb] = s;"),
    "GEMM uses the first group's x scale": ("xhat[k] = e4m3_signed(xq[m * K + k]) * xs_at(m, k / block);",
                                            "xhat[k] = e4m3_signed(xq[m * K + k]) * xs_at(m, 0);"),
    "GEMM drops the bias": ("if (bias) acc += static_cast<double>(bf16_to_float(bias[n]));", "if (bias) acc += 0.0;"),
    "GEMM bound without magnitudes": ("mag += std::fabs(p);", "mag += p;"),
    "GEMM drops the last k": ("for (int64_t k = 0; k < K; ++k) {\n        const double p",
                              "for (int64_t k = 0; k < K - 1; ++k) {\n        const double p"),
    "bf16 output truncated": ("const double r = std::nearbyint(scaled);", "const double r = std::floor(scaled);"),
    "dequant ignores the column block": ("const int64_t blk = (n / kBlock) * Kb + k / kBlock;",
                                         "const int64_t blk = (n / kBlock) * Kb;"),
    "static scale multiplies": ("xq[m * K + k] = e4m3_encode(bf16_to_float(x[m * ld_x + k]) / s);",
                                "xq[m * K + k] = e4m3_encode(bf16_to_float(x[m * ld_x + k]) * s);"),
    "1 x 32 groups span 128 channels": ("const int64_t k1 = std::min<int64_t>(k0 + group, K);",
                                        "const int64_t k1 = std::min<int64_t>(k0 + kGroup, K);"),
    "GEMM weight row block fixed at 128": ("ws_at(n / block, k / block)", "ws_at(n / kBlock, k / block)"),
    "e4m3 subnormals off by a factor 2": ("mag = std::ldexp(static_cast<double>(mant), -9);",
                                          "mag = std::ldexp(static_cast<double>(mant), -10);"),
    "scale conversion accepts non-powers": ("if (f == 0.5 && e >= -127 && e <= 127)", "if (e >= -127 && e <= 127)"),
    "bf16 subnormal quantum off by one": ("if (q < -133) q = -133;", "if (q < -132) q = -132;"),
    "GEMM decode drops the sign": ("return (code & 0x80) ? -mag : mag;", "return mag;"),
    "sampled rows read from the top": ("const int64_t m = rows ? rows[r] : r;\n    std::vector<double> xhat",
                                       "const int64_t m = r;\n    std::vector<double> xhat"),
}


# Python grouped layer (oracle/__init__.py): name: (text, planted replacement)
PY_MUTATIONS = {
    "grouped tile of 64 rows": ("MOE_TILE = 128", "MOE_TILE = 64"),
    "grouped expert from the block's last row": ("        e = int(re[t * MOE_TILE])\n",
                                                 "        e = int(re[min(M, (t + 1) * MOE_TILE) - 1])\n"),
    "grouped -1 blocks computed with expert 0": ("        if e < 0:\n            continue\n",
                                                 "        if e < 0:\n            e = 0\n"),
    "grouped bias of expert 0": ("None if bias_bf16 is None else bias_bf16[e], fmt, rows=rows)",
                                 "None if bias_bf16 is None else bias_bf16[0], fmt, rows=rows)"),
    "grouped scales of expert 0": ("wq[e], ws[e],", "wq[e], ws[0],"),
}


def _py_tree(tmp, i, name):
    """A copy of the oracle, tests and input generators with one Python mistake planted."""
    root = os.path.join(tmp, f"tree{i}")
    skip = shutil.ignore_patterns("__pycache__", "*.so", "*.so.tmp")
    for d in ("oracle", "tests", "workloads"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(root, d), ignore=skip)
    shutil.copy(os.path.join(ROOT, "pytest.ini"), root)
    if name is not None:
        path = os.path.join(root, "oracle", "__init__.py")
        src = open(path).read()
        old, new = PY_MUTATIONS[name]
        assert src.count(old) == 1, f"{name}: the text to mutate is not unique in the oracle's Python"
        with open(path, "w") as f:
            f.write(src.replace(old, new))
    return root


def _build(tmp, i, name):
    from oracle import build
    src = open(SRC).read()
    if name is not None:
        old, new = MUTATIONS[name]
        assert src.count(old) == 1, f"{name}: the text to mutate is not unique in the oracle source"
        src = src.replace(old, new)
    path = os.path.join(tmp, f"m{i}.cpp")
    with open(path, "w") as f:
        f.write(src)
    return build.compile_library(path, os.path.join(tmp, f"libm{i}.so"))


def _run_pins(lib, root=ROOT):
    env = dict(os.environ, FG8_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(root, "tests", "test_oracle.py"), "-x", "-q",
                        "-p", "no:cacheprovider", "-m", "not gpu"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-600:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    from oracle import build
    names = [None] + list(MUTATIONS)
    with concurrent.futures.ThreadPoolExecutor(4) as pool:
        libs = list(pool.map(lambda a: _build(str(tmp_path), *a), enumerate(names)))
        py_names = ["tree control"] + list(PY_MUTATIONS)
        trees = [_py_tree(str(tmp_path), i, None if i == 0 else n) for i, n in enumerate(py_names)]
        results = dict(zip(names, pool.map(_run_pins, libs)))
        real = build.build()
        results.update(zip(py_names, pool.map(lambda t: _run_pins(real, t), trees)))
    for control in (None, "tree control"):
        rc, out = results[control]
        assert rc == 0, f"an unmodified copy ({control or 'compiled'}) must pass every pin:\n{out}"
    # pytest exit status 1: some test failed (not a crash, a usage error or an empty run)
    survivors = {n: results[n] for n in list(MUTATIONS) + list(PY_MUTATIONS) if results[n][0] != 1}
    assert not survivors, "planted mistakes no pin caught: " + "; ".join(
        f"{n} (exit {rc})" for n, (rc, _) in survivors.items())
