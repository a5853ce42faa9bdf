"""Decode what fg8_linear_prepare (or a chained GEMM's epilogue) leaves in a
layer's workspace, so the tests can compare it with the oracle's row-major
codes and scales.

The layout is the one include/fg8.h documents for fg8_linear's workspace:
a 1024-byte header, then the e4m3 codes [M, K] (row stride K), then, 256-byte
aligned, the activation scales in the GEMM's layout:
  float  K-major [ceil(K/128)][ld_s] float32 with ld_s = M rounded up to 256;
  UE8M0  scale-factor tiles of 128 rows x 4 K-blocks (512 bytes each): tile
         (r // 128, kb // 4) at ((r // 128) * Kq + kb // 4) * 512, inside it
         the word of row 32c + i at i * 16 + c * 4, byte kb % 4.
This module only reads bytes back; it computes nothing of the method.
"""
import numpy as np

HEADER = 1024
ALIGN = 256


def _align(v, a=ALIGN):
    return (v + a - 1) // a * a


def offsets(M, K):
    """(xq offset, scale offset, ld_s) of fg8_linear's workspace for M tokens and K channels."""
    xq_off = HEADER
    xs_off = _align(xq_off + M * K)
    ld_s = _align(M, 256)
    return xq_off, xs_off, ld_s


def sf_tile_offsets(M, Kb):
    """[M, Kb] byte offsets of every (row, K-block) UE8M0 scale inside the scale-factor tiles."""
    Kq = (Kb + 3) // 4
    r = np.arange(M, dtype=np.int64)[:, None]
    kb = np.arange(Kb, dtype=np.int64)[None, :]
    rr = r % 128
    return ((r // 128) * Kq + kb // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + (kb % 4)


def decode(ws_bytes, M, K, fmt):
    """Workspace bytes (numpy uint8) -> (xq [M, K] uint8, scales [M, ceil(K/128)] as
    uint32 bit patterns (float) or uint8 bytes (UE8M0))."""
    Kb = (K + 127) // 128
    xq_off, xs_off, ld_s = offsets(M, K)
    xq = ws_bytes[xq_off:xq_off + M * K].reshape(M, K)
    if fmt == 0:
        kmaj = ws_bytes[xs_off:xs_off + Kb * ld_s * 4].view(np.uint32).reshape(Kb, ld_s)
        xs = np.ascontiguousarray(kmaj[:, :M].T)
    else:
        xs = ws_bytes[xs_off + sf_tile_offsets(M, Kb)]
    return xq, xs
