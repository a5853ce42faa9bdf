"""CPU oracle for the fine-grained FP8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (the CUDA library and its Python
binding) never imports, loads or calls it, and it shares no code with them.

The arithmetic lives in ``fg8_oracle.cpp`` (plain C++, float32 scales and
quotients, double accumulation); this module only marshals numpy arrays.
bf16 data is passed as ``uint16`` bit patterns, e4m3fn and UE8M0 as ``uint8``.

Sources: [zh] "Transformers 中的细粒度 FP8 量化：配置、DeepGEMM 加速路径与 UE8M0
缩放格式完全指南" and [pt] "FP8 de granularidade fina".  The quantizers follow
[zh] §一 (1x128 per-token activation groups, 128x128 weight blocks,
weight_scale_inv shaped (ceil(out/128), ceil(in/128))) and [zh] §七 (UE8M0
scales); the GEMM follows [zh] §八 step 6 (FP8Linear.forward -> fp8_linear).
"""
import ctypes
import os

import numpy as np

from . import build as _build

FMT_FLOAT = 0
FMT_UE8M0 = 1
GROUP = 128

_lib = None


def lib():
    global _lib
    if _lib is None:
        # FG8_ORACLE_LIB: a library compiled from another copy of the source
        # (the mutation tests load deliberately broken copies this way)
        path = os.environ.get("FG8_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        c_u8p = ctypes.POINTER(ctypes.c_uint8)
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_num_threads.argtypes = []
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e8m0_value.restype = ctypes.c_float
        L.orc_e8m0_value.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_ceil_byte.restype = ctypes.c_uint8
        L.orc_e8m0_ceil_byte.argtypes = [ctypes.c_float]
        L.orc_group_scale.restype = ctypes.c_float
        L.orc_group_scale.argtypes = [ctypes.c_float]
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_bf16_from_double.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode_many.restype = None
        L.orc_e4m3_encode_many.argtypes = [ctypes.c_void_p, ctypes.c_int64, c_u8p]
        for name in ("orc_quantize_act", "orc_quantize_weight"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                          ctypes.c_void_p, ctypes.c_void_p]
        L.orc_linear_dequant.restype = ctypes.c_int
        for name in ("orc_quantize_act_g", "orc_quantize_weight_b"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                          ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_linear_dequant_b.restype = ctypes.c_int
        L.orc_linear_dequant_b.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_dequantize_weight.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                            ctypes.c_int, ctypes.c_void_p, ctypes.c_int64]
        L.orc_dequantize_weight.restype = ctypes.c_int
        L.orc_quantize_act_static.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_float, ctypes.c_void_p]
        L.orc_quantize_act_static.restype = ctypes.c_int
        L.orc_scale_to_e8m0.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_scale_to_e8m0.restype = ctypes.c_int64
        L.orc_linear_dequant.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p]
        _lib = L
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _nb(k, block):
    return -(-k // block)


def _kb(k):
    return (k + GROUP - 1) // GROUP


def _scale_dtype(fmt):
    return np.float32 if fmt == FMT_FLOAT else np.uint8


# ---------------------------------------------------------------- scalars --
def num_threads() -> int:
    """Host threads the oracle's OpenMP loops run on."""
    return int(lib().orc_num_threads())


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(int(code))


def e4m3_encode(f: float) -> int:
    return int(lib().orc_e4m3_encode(float(np.float32(f))))


def e4m3_encode_many(f: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32).ravel()
    out = np.empty(f.size, dtype=np.uint8)
    lib().orc_e4m3_encode_many(_ptr(f), f.size, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out


def e8m0_value(b: int) -> float:
    return float(lib().orc_e8m0_value(int(b)))


def e8m0_ceil_byte(s: float) -> int:
    return int(lib().orc_e8m0_ceil_byte(float(np.float32(s))))


def group_scale(amax: float) -> float:
    return float(np.float32(lib().orc_group_scale(float(np.float32(amax)))))


def bf16_from_double(v: float) -> int:
    return int(lib().orc_bf16_from_double(float(v)))


# ------------------------------------------------------------- quantizers --
def quantize_act(x_bf16: np.ndarray, fmt: int, block: int = GROUP):
    """x bf16 bits [M, K] -> (xq e4m3 [M, K], x_scale [M, ceil(K/block)] float32|uint8).

    block: the group width (the weight block's input-channel size; 128 by
    default, [zh] §一; other block sizes such as (32, 32) are tested
    configurations on the pages, [zh] §八)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    xq = np.empty((M, K), dtype=np.uint8)
    xs = np.empty((M, _nb(K, block)), dtype=_scale_dtype(fmt))
    rc = lib().orc_quantize_act_g(_ptr(x), M, K, K, fmt, block, _ptr(xq), _ptr(xs))
    if rc != 0:
        raise ValueError("orc_quantize_act: bad argument")
    return xq, xs


def quantize_act_static(x_bf16: np.ndarray, scale: float):
    """Static scheme: x bf16 bits [M, K] and one float32 scale -> (xq e4m3 [M, K],
    x_scale [M, ceil(K/128)] float32 all equal to the scale, the GEMM's view)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    xq = np.empty((M, K), dtype=np.uint8)
    if lib().orc_quantize_act_static(_ptr(x), M, K, K, float(np.float32(scale)), _ptr(xq)) != 0:
        raise ValueError("orc_quantize_act_static: bad argument")
    return xq, np.full((M, _kb(K)), np.float32(scale), dtype=np.float32)


def quantize_weight(w_bf16: np.ndarray, fmt: int, block: int = GROUP):
    """W bf16 bits [N, K] -> (wq e4m3 [N, K], w_scale_inv [ceil(N/block), ceil(K/block)]);
    block x block weight blocks (128 by default)."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    wq = np.empty((N, K), dtype=np.uint8)
    ws = np.empty((_nb(N, block), _nb(K, block)), dtype=_scale_dtype(fmt))
    rc = lib().orc_quantize_weight_b(_ptr(w), N, K, K, fmt, block, _ptr(wq), _ptr(ws))
    if rc != 0:
        raise ValueError("orc_quantize_weight: bad argument")
    return wq, ws


def linear_dequant(xq, xs, wq, ws, bias_bf16, fmt, rows=None, block: int = GROUP):
    """Reference y for quantized operands.

    Returns (y64 [R, N] float64, bound [R, N] float64, y_bf16 [R, N] uint16),
    R = len(rows) (or M when rows is None).
    """
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    xs = np.ascontiguousarray(xs, dtype=_scale_dtype(fmt))
    ws = np.ascontiguousarray(ws, dtype=_scale_dtype(fmt))
    M, K = xq.shape
    N, K2 = wq.shape
    if K2 != K:
        raise ValueError("K mismatch")
    if xs.shape != (M, _nb(K, block)) or ws.shape != (_nb(N, block), _nb(K, block)):
        raise ValueError("scale shape mismatch")
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    if b is not None and b.shape != (N,):
        raise ValueError("bias shape mismatch")
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    R = M if r is None else r.size
    y64 = np.empty((R, N), dtype=np.float64)
    bound = np.empty((R, N), dtype=np.float64)
    ybf = np.empty((R, N), dtype=np.uint16)
    rc = lib().orc_linear_dequant_b(_ptr(xq), _ptr(xs), _ptr(wq), _ptr(ws), _ptr(b), M, N, K, fmt, block,
                                    _ptr(r), 0 if r is None else r.size, _ptr(y64), _ptr(bound), _ptr(ybf))
    if rc != 0:
        raise ValueError("orc_linear_dequant: bad argument")
    return y64, bound, ybf


def linear(x_bf16, wq, ws, bias_bf16, fmt, rows=None, block: int = GROUP):
    """Whole layer: quantize x per token (1 x block groups), then linear_dequant
    with block x block weight blocks."""
    xq, xs = quantize_act(x_bf16, fmt, block)
    return linear_dequant(xq, xs, wq, ws, bias_bf16, fmt, rows, block)


# ------------------------------------------------------ MoE experts ------
MOE_TILE = 128  # rows of one expert block in the contiguous grouped layout


def grouped_linear(x_bf16, row_expert, wq, ws, bias_bf16, fmt):
    """The expert GEMM of an MoE layer ([zh] §6.4 / [pt] "Caminho rápido do
    DeepGEMM": FP8Experts sends each expert's tokens through the fine-grained
    FP8 linear of [zh] §八 step 6, with that expert's e4m3 weights and block
    scales; on Blackwell the expert kernels take UE8M0 scales).

    Layout (a reading: the pages print no expert kernel interface): the
    routed rows of x are sorted by expert, each expert's run padded to whole
    blocks of MOE_TILE rows; block t = rows [128 t, 128 t + 128) is computed
    with expert row_expert[128 t], and skipped when that is -1.  The
    activation groups are per token, so x is quantized once for all experts.

    x_bf16 [M, K] (bits), row_expert [M] int, wq [E, N, K], ws [E, Nb, Kb],
    bias_bf16 [E, N] or None.  Returns (y64, bound, y_bf16, written): rows of
    skipped blocks have written False, y64 NaN and y_bf16 0.
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    re = np.asarray(row_expert).astype(np.int64)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    ws = np.ascontiguousarray(ws, dtype=_scale_dtype(fmt))
    M, K = x.shape
    E, N, K2 = wq.shape
    if K2 != K or re.shape != (M,) or ws.shape != (E, _kb(N), _kb(K)):
        raise ValueError("shape mismatch")
    if bias_bf16 is not None and np.shape(bias_bf16) != (E, N):
        raise ValueError("bias shape mismatch")
    xq, xs = quantize_act(x, fmt)
    y64 = np.full((M, N), np.nan)
    bound = np.zeros((M, N))
    ybf = np.zeros((M, N), dtype=np.uint16)
    written = np.zeros(M, dtype=bool)
    for t in range(-(-M // MOE_TILE)):
        e = int(re[t * MOE_TILE])
        if e < 0:
            continue
        if e >= E:
            raise ValueError(f"block {t}: expert {e} >= {E}")
        rows = np.arange(t * MOE_TILE, min(M, (t + 1) * MOE_TILE))
        a, b, c = linear_dequant(xq, xs, wq[e], ws[e], None if bias_bf16 is None else bias_bf16[e], fmt, rows=rows)
        y64[rows], bound[rows], ybf[rows], written[rows] = a, b, c, True
    return y64, bound, ybf, written


# ------------------------------------------------ checkpoint conversions --
def dequantize_weight(wq, ws, fmt: int) -> np.ndarray:
    """Fp8Dequantize: e4m3 [N, K] and its block scales -> bf16 bits [N, K]."""
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    ws = np.ascontiguousarray(ws, dtype=_scale_dtype(fmt))
    N, K = wq.shape
    if ws.shape != (_kb(N), _kb(K)):
        raise ValueError("scale shape mismatch")
    w = np.empty((N, K), dtype=np.uint16)
    if lib().orc_dequantize_weight(_ptr(wq), N, K, _ptr(ws), fmt, _ptr(w), K) != 0:
        raise ValueError("orc_dequantize_weight: bad argument")
    return w


def scale_to_e8m0(s) -> tuple:
    """float32 power-of-two scales -> (UE8M0 bytes, number of inputs that were no UE8M0 value)."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.empty(s.shape, dtype=np.uint8)
    bad = lib().orc_scale_to_e8m0(_ptr(s), s.size, _ptr(out))
    return out, int(bad)
