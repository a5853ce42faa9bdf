"""B200 (sm_100a) fine-grained FP8 linear layer.

A thin Python binding over ``libfg8.so`` (C ABI: ``include/fg8.h``).  Every
step of the layer runs in the library's CUDA kernels; this module only
marshals arguments.  PyTorch supplies device memory and the current stream.
There is no CPU or PyTorch fallback: if the library is missing or the device
is not a B200, calls raise.

The method is the one the Transformers fine-grained FP8 pages describe
("Transformers 中的细粒度 FP8 量化：配置、DeepGEMM 加速路径与 UE8M0 缩放格式完全指南",
§一 / §七 / §八; "FP8 de granularidade fina"): 128x128 e4m3 weight blocks,
per-token 1x128 dynamic activation groups, float32 or UE8M0 scales,
y = dequant(xq) . dequant(Wq)^T + bias in bf16.
"""
from ._capi import (  # noqa: F401  (re-exported C ABI)
    FG8_ERR_ALIGNMENT,
    FG8_ERR_CUDA,
    FG8_ERR_INVALID_ARG,
    FG8_ERR_TIMEOUT,
    FG8_ERR_UNSUPPORTED_DEVICE,
    FG8_ERR_WORKSPACE,
    FG8_OK,
    FG8_SCALE_FLOAT,
    FG8_SCALE_UE8M0,
    FG8Error,
    fg8_check_device_status,
    fg8_dequantize_weight,
    fg8_gemm_prequant,
    fg8_gemm_workspace_bytes,
    fg8_grouped_linear,
    fg8_grouped_linear_prepare,
    fg8_grouped_linear_run,
    fg8_grouped_row_expert,
    fg8_grouped_linear_workspace_bytes,
    fg8_linear,
    fg8_linear_block,
    fg8_linear_block_workspace_bytes,
    fg8_linear_fused,
    fg8_linear_fused_workspace_bytes,
    fg8_linear_noalloc,
    fg8_linear_prepare,
    fg8_linear_run,
    fg8_linear_run_chain,
    fg8_linear_static,
    fg8_linear_workspace_bytes,
    fg8_linear_plan,
    fg8_quantize_act,
    fg8_quantize_act_block,
    fg8_quantize_act_static,
    fg8_quantize_weight,
    fg8_quantize_weight_block,
    fg8_scale_to_ue8m0,
    fg8_set_test_stall,
    fg8_set_wait_limit_ns,
    fg8_status_string,
    fg8_version,
    lib,
    library_path,
)
from .layer import (  # noqa: F401
    FP8Linear,
    dequantize_weight,
    gemm_prequant,
    grouped_linear,
    linear,
    linear_chain,
    linear_static,
    quantize_act,
    quantize_act_static,
    quantize_weight,
    scale_fmt_code,
    scale_to_ue8m0,
)
