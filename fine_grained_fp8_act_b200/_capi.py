"""ctypes binding of libfg8.so: the C ABI of include/fg8.h, same names.

Pointers are plain integers (device addresses), sizes are int64, `stream` is
a cudaStream_t handle as an integer.  Each wrapper raises FG8Error on a
non-zero status; nothing here computes.
"""
import ctypes
import os

FG8_SCALE_FLOAT = 0
FG8_SCALE_UE8M0 = 1

FG8_OK = 0
FG8_ERR_INVALID_ARG = 1
FG8_ERR_ALIGNMENT = 2
FG8_ERR_UNSUPPORTED_DEVICE = 3
FG8_ERR_WORKSPACE = 4
FG8_ERR_CUDA = 5
FG8_ERR_TIMEOUT = 6

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfg8.so")
_lib = None

_VP = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes), exactly the declarations of include/fg8.h
SIGNATURES = {
    "fg8_quantize_weight": (_INT, [_VP, _I64, _I64, _I64, _VP, _VP, _INT, _VP]),
    "fg8_quantize_act": (_INT, [_VP, _I64, _I64, _I64, _VP, _VP, _INT, _VP]),
    "fg8_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64, _INT]),
    "fg8_linear_plan": (_INT, [_I64, _I64, _I64, _INT, _VP]),
    "fg8_linear": (_INT, [_VP, _I64, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _I64, _INT, _VP, _SZ, _VP]),
    "fg8_linear_prepare": (_INT, [_VP, _I64, _I64, _I64, _I64, _VP, _INT, _VP, _SZ, _VP]),
    "fg8_grouped_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I64, _INT]),
    "fg8_grouped_linear": (_INT, [_VP, _I64, _I64, _I64, _VP, _I64, _I64, _VP, _VP, _VP, _VP, _I64, _INT, _VP, _SZ,
                                  _VP]),
    "fg8_grouped_linear_prepare": (_INT, [_VP, _I64, _I64, _I64, _I64, _I64, _VP, _INT, _VP, _SZ, _VP]),
    "fg8_grouped_linear_run": (_INT, [_VP, _I64, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _I64, _INT, _VP, _SZ, _VP]),
    "fg8_quantize_act_block": (_INT, [_VP, _I64, _I64, _I64, _VP, _VP, _INT, _INT, _VP]),
    "fg8_quantize_weight_block": (_INT, [_VP, _I64, _I64, _I64, _VP, _VP, _INT, _INT, _VP]),
    "fg8_linear_block_workspace_bytes": (_SZ, [_I64, _I64, _I64, _INT, _INT]),
    "fg8_linear_block": (_INT, [_VP, _I64, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _I64, _INT, _INT, _VP, _SZ, _VP]),
    "fg8_grouped_row_expert": (_INT, [_VP, _I64, _I64, _VP, _VP]),
    "fg8_linear_run": (_INT, [_VP, _VP, _VP, _VP, _I64, _I64, _I64, _I64, _INT, _VP, _SZ, _VP]),
    "fg8_linear_run_chain": (_INT, [_VP, _VP, _VP, _VP, _I64, _I64, _I64, _I64, _INT, _VP, _SZ, _I64, _VP, _VP, _SZ,
                                     _VP]),
    "fg8_linear_noalloc": (_INT, [_VP, _I64, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _I64, _INT, _VP]),
    "fg8_linear_fused_workspace_bytes": (_SZ, [_I64, _I64, _I64, _INT]),
    "fg8_linear_fused": (_INT, [_VP, _I64, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _I64, _INT, _VP, _SZ, _I64, _VP,
                                _VP, _SZ, _VP]),
    "fg8_gemm_workspace_bytes": (_SZ, [_I64, _I64, _I64, _INT]),
    "fg8_gemm_prequant": (_INT, [_VP, _VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _I64, _INT, _VP, _SZ, _VP]),
    "fg8_quantize_act_static": (_INT, [_VP, _I64, _I64, _I64, _VP, _VP, _VP, _VP]),
    "fg8_linear_static": (_INT, [_VP, _I64, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _I64, _VP, _SZ, _VP]),
    "fg8_dequantize_weight": (_INT, [_VP, _I64, _I64, _VP, _INT, _VP, _I64, _VP]),
    "fg8_scale_to_ue8m0": (_INT, [_VP, _I64, _VP, _VP, _VP]),
    "fg8_check_device_status": (_INT, [_VP, _VP]),
    "fg8_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "fg8_set_test_stall": (None, [_INT]),
    "fg8_status_string": (ctypes.c_char_p, [_INT]),
    "fg8_version": (_INT, []),
}


class FG8Error(RuntimeError):
    def __init__(self, func, status):
        self.status = int(status)
        super().__init__(f"{func}: status {self.status} ({fg8_status_string(self.status)})")


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libfg8.so once.  Raises if it has not been built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m fine_grained_fp8_act_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(func, status):
    if status != FG8_OK:
        raise FG8Error(func, status)


def fg8_status_string(status: int) -> str:
    return lib().fg8_status_string(int(status)).decode()


def fg8_version() -> int:
    return lib().fg8_version()


def fg8_set_wait_limit_ns(ns: int) -> None:
    lib().fg8_set_wait_limit_ns(int(ns))


def fg8_set_test_stall(on: bool) -> None:
    lib().fg8_set_test_stall(1 if on else 0)


def fg8_quantize_weight(w_bf16, N, K, ld_w, wq_e4m3, w_scale_inv, fmt, stream):
    _check("fg8_quantize_weight", lib().fg8_quantize_weight(w_bf16, N, K, ld_w, wq_e4m3, w_scale_inv, fmt, stream))


def fg8_quantize_act(x_bf16, M, K, ld_x, xq_e4m3, x_scale, fmt, stream):
    _check("fg8_quantize_act", lib().fg8_quantize_act(x_bf16, M, K, ld_x, xq_e4m3, x_scale, fmt, stream))


def fg8_linear_workspace_bytes(M, N, K, fmt) -> int:
    return int(lib().fg8_linear_workspace_bytes(M, N, K, fmt))


def fg8_linear_plan(M, N, K, fmt):
    """(kernel, tile width, split tiles, units per split tile): how fg8_linear runs
    this shape on the current device; see include/fg8.h."""
    out = (ctypes.c_int32 * 4)()
    _check("fg8_linear_plan", lib().fg8_linear_plan(M, N, K, fmt, out))
    return tuple(int(v) for v in out)


def fg8_gemm_workspace_bytes(M, N, K, fmt) -> int:
    return int(lib().fg8_gemm_workspace_bytes(M, N, K, fmt))


def fg8_linear(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, workspace,
               workspace_bytes, stream):
    _check("fg8_linear", lib().fg8_linear(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt,
                                          workspace, workspace_bytes, stream))


def fg8_linear_prepare(x_bf16, M, N, K, ld_x, w_scale_inv, fmt, workspace, workspace_bytes, stream):
    _check("fg8_linear_prepare", lib().fg8_linear_prepare(x_bf16, M, N, K, ld_x, w_scale_inv, fmt, workspace,
                                                          workspace_bytes, stream))


def fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt):
    return lib().fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt)


def fg8_grouped_linear(x_bf16, M, K, ld_x, row_expert, E, N, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt,
                       workspace, workspace_bytes, stream):
    _check("fg8_grouped_linear", lib().fg8_grouped_linear(x_bf16, M, K, ld_x, row_expert, E, N, wq_e4m3, w_scale_inv,
                                                          bias_bf16, y_bf16, ld_y, fmt, workspace, workspace_bytes,
                                                          stream))


def fg8_grouped_linear_prepare(x_bf16, M, K, ld_x, E, N, w_scale_inv, fmt, workspace, workspace_bytes, stream):
    _check("fg8_grouped_linear_prepare", lib().fg8_grouped_linear_prepare(x_bf16, M, K, ld_x, E, N, w_scale_inv, fmt,
                                                                          workspace, workspace_bytes, stream))


def fg8_grouped_linear_run(row_expert, E, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace,
                           workspace_bytes, stream):
    _check("fg8_grouped_linear_run", lib().fg8_grouped_linear_run(row_expert, E, wq_e4m3, w_scale_inv, bias_bf16,
                                                                  y_bf16, M, N, K, ld_y, fmt, workspace,
                                                                  workspace_bytes, stream))


def fg8_quantize_act_block(x_bf16, M, K, ld_x, xq_e4m3, x_scale, fmt, block, stream):
    _check("fg8_quantize_act_block", lib().fg8_quantize_act_block(x_bf16, M, K, ld_x, xq_e4m3, x_scale, fmt, block,
                                                                  stream))


def fg8_quantize_weight_block(w_bf16, N, K, ld_w, wq_e4m3, w_scale_inv, fmt, block, stream):
    _check("fg8_quantize_weight_block", lib().fg8_quantize_weight_block(w_bf16, N, K, ld_w, wq_e4m3, w_scale_inv, fmt,
                                                                        block, stream))


def fg8_linear_block_workspace_bytes(M, N, K, fmt, block):
    return lib().fg8_linear_block_workspace_bytes(M, N, K, fmt, block)


def fg8_linear_block(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, block, workspace,
                     workspace_bytes, stream):
    _check("fg8_linear_block", lib().fg8_linear_block(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16,
                                                      ld_y, fmt, block, workspace, workspace_bytes, stream))


def fg8_grouped_row_expert(counts, E, cap, row_expert, stream):
    _check("fg8_grouped_row_expert", lib().fg8_grouped_row_expert(counts, E, cap, row_expert, stream))


def fg8_linear_run(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace, workspace_bytes, stream):
    _check("fg8_linear_run", lib().fg8_linear_run(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt,
                                                  workspace, workspace_bytes, stream))


def fg8_linear_run_chain(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace, workspace_bytes,
                         next_N, next_w_scale_inv, next_workspace, next_workspace_bytes, stream):
    _check("fg8_linear_run_chain", lib().fg8_linear_run_chain(wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y,
                                                              fmt, workspace, workspace_bytes, next_N,
                                                              next_w_scale_inv, next_workspace, next_workspace_bytes,
                                                              stream))


def fg8_linear_fused_workspace_bytes(M, N, K, fmt) -> int:
    return int(lib().fg8_linear_fused_workspace_bytes(M, N, K, fmt))


def fg8_linear_fused(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, workspace,
                     workspace_bytes, next_N=0, next_w_scale_inv=None, next_workspace=None, next_workspace_bytes=0,
                     stream=None):
    """fg8_linear with the activation quantization inside the GEMM kernel (optionally
    also quantizing y for a next layer, as fg8_linear_run_chain)."""
    _check("fg8_linear_fused", lib().fg8_linear_fused(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16,
                                                      ld_y, fmt, workspace, workspace_bytes, next_N,
                                                      next_w_scale_inv, next_workspace, next_workspace_bytes, stream))


def fg8_linear_noalloc(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, fmt, stream):
    """fg8_linear with the library's fixed device scratch instead of a caller workspace."""
    _check("fg8_linear_noalloc", lib().fg8_linear_noalloc(x_bf16, M, N, K, ld_x, wq_e4m3, w_scale_inv, bias_bf16,
                                                          y_bf16, ld_y, fmt, stream))


def fg8_gemm_prequant(xq_e4m3, x_scale, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M, N, K, ld_y, fmt, workspace,
                      workspace_bytes, stream):
    _check("fg8_gemm_prequant", lib().fg8_gemm_prequant(xq_e4m3, x_scale, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, M,
                                                        N, K, ld_y, fmt, workspace, workspace_bytes, stream))


def fg8_quantize_act_static(x_bf16, M, K, ld_x, act_scale, xq_e4m3, x_scale, stream):
    _check("fg8_quantize_act_static", lib().fg8_quantize_act_static(x_bf16, M, K, ld_x, act_scale, xq_e4m3, x_scale,
                                                                    stream))


def fg8_linear_static(x_bf16, M, N, K, ld_x, act_scale, wq_e4m3, w_scale_inv, bias_bf16, y_bf16, ld_y, workspace,
                      workspace_bytes, stream):
    _check("fg8_linear_static", lib().fg8_linear_static(x_bf16, M, N, K, ld_x, act_scale, wq_e4m3, w_scale_inv,
                                                        bias_bf16, y_bf16, ld_y, workspace, workspace_bytes, stream))


def fg8_dequantize_weight(wq_e4m3, N, K, w_scale_inv, fmt, w_bf16, ld_w, stream):
    _check("fg8_dequantize_weight", lib().fg8_dequantize_weight(wq_e4m3, N, K, w_scale_inv, fmt, w_bf16, ld_w, stream))


def fg8_scale_to_ue8m0(scale_f32, n, scale_e8m0, invalid_count, stream):
    _check("fg8_scale_to_ue8m0", lib().fg8_scale_to_ue8m0(scale_f32, n, scale_e8m0, invalid_count, stream))


def fg8_check_device_status(workspace, stream) -> int:
    """Returns the status code the previous calls on this workspace left: FG8_OK,
    FG8_ERR_TIMEOUT, or FG8_ERR_INVALID_ARG for an expert index >= E in a
    grouped call; synchronizes the stream and clears the word; does not raise."""
    return int(lib().fg8_check_device_status(workspace, stream))
