"""PyTorch-facing wrappers: tensors in, tensors out, through the C ABI.

These functions allocate outputs with torch on the input's device, pass raw
pointers and the current CUDA stream to libfg8, and return.  They do no
arithmetic of their own.

Storage follows the Transformers fine-grained FP8 page ("Transformers 中的细粒度
FP8 量化 ... 完全指南", §一 and §七): weights as torch.float8_e4m3fn, one
weight_scale_inv per 128x128 block shaped (ceil(out/128), ceil(in/128)),
float32 or torch.float8_e8m0fnu for scale_fmt "ue8m0".
"""
from typing import Optional, Tuple

import torch

from . import _capi as C

_SCALE_DTYPES = {C.FG8_SCALE_FLOAT: torch.float32, C.FG8_SCALE_UE8M0: torch.float8_e8m0fnu}


def scale_fmt_code(scale_fmt) -> int:
    """"float" -> 0, "ue8m0" -> 1 (the only two values [zh] §四 accepts)."""
    if isinstance(scale_fmt, int) and scale_fmt in (C.FG8_SCALE_FLOAT, C.FG8_SCALE_UE8M0):
        return scale_fmt
    if scale_fmt == "float":
        return C.FG8_SCALE_FLOAT
    if scale_fmt == "ue8m0":
        return C.FG8_SCALE_UE8M0
    raise ValueError(f"scale_fmt must be 'float' or 'ue8m0', got {scale_fmt!r}")


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _cdiv(a: int, b: int) -> int:
    return (a + b - 1) // b


# The C ABI takes raw pointers and cannot see how large a buffer is, so every
# operand a kernel reads or writes is checked here against the shape, dtype and
# device the call implies before its pointer is passed on.  e4m3 codes and UE8M0
# scales may also come as raw uint8 bytes (the same bits).
_E4M3 = (torch.float8_e4m3fn, torch.uint8)


def _scale_dtypes(fmt: int):
    return (torch.float32,) if fmt == C.FG8_SCALE_FLOAT else (torch.float8_e8m0fnu, torch.uint8)


def _check_bf16_matrix(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.dim() != 2:
        raise ValueError(f"{name} must be a 2-D bf16 tensor")
    if t.stride(1) != 1 or (t.shape[0] > 1 and t.stride(0) < t.shape[1]):
        raise ValueError(f"{name} must have unit stride in its last dimension and rows that do not overlap")


def _check_cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _check_tensor(t, name: str, shape, dtypes, device):
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must be {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_weight(wq, w_scale_inv, lead, N: int, K: int, fmt: int, block: int, device):
    """wq e4m3 [*lead, N, K] and its block scales [*lead, ceil(N/block), ceil(K/block)]."""
    _check_tensor(wq, "wq", (*lead, N, K), _E4M3, device)
    _check_tensor(w_scale_inv, "w_scale_inv", (*lead, _cdiv(N, block), _cdiv(K, block)), _scale_dtypes(fmt), device)


def _check_bias(bias, shape, device) -> int:
    if bias is None:
        return 0
    _check_tensor(bias, "bias", shape, (torch.bfloat16,), device)
    return bias.data_ptr()


def _output(out, M: int, N: int, device) -> torch.Tensor:
    """out as given (bf16 [M, N], unit column stride, row stride >= N) or a new tensor."""
    if out is None:
        return torch.empty((M, N), dtype=torch.bfloat16, device=device)
    _check_bf16_matrix(out, "out")
    if tuple(out.shape) != (M, N) or out.device != device:
        raise ValueError(f"out must be [{M}, {N}] on {device}")
    return out


def quantize_weight(w: torch.Tensor, scale_fmt="float", block: int = 128) -> Tuple[torch.Tensor, torch.Tensor]:
    """W bf16 [N, K] -> (wq float8_e4m3fn [N, K], weight_scale_inv [ceil(N/block), ceil(K/block)]);
    block x block weight blocks, block 128 (default), 64 or 32."""
    fmt = scale_fmt_code(scale_fmt)
    _check_bf16_matrix(w, "w")
    _check_cuda(w, "w")
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    ws = torch.empty((_cdiv(N, block), _cdiv(K, block)), dtype=_SCALE_DTYPES[fmt], device=w.device)
    with torch.cuda.device(w.device):
        C.fg8_quantize_weight_block(w.data_ptr(), N, K, w.stride(0), wq.data_ptr(), ws.data_ptr(), fmt, block,
                                    _stream(w))
    return wq, ws


def quantize_act(x: torch.Tensor, scale_fmt="float", block: int = 128) -> Tuple[torch.Tensor, torch.Tensor]:
    """x bf16 [M, K] -> (xq float8_e4m3fn [M, K], x_scale [M, ceil(K/block)]); 1 x block groups."""
    fmt = scale_fmt_code(scale_fmt)
    _check_bf16_matrix(x, "x")
    _check_cuda(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    xs = torch.empty((M, _cdiv(K, block)), dtype=_SCALE_DTYPES[fmt], device=x.device)
    with torch.cuda.device(x.device):
        C.fg8_quantize_act_block(x.data_ptr(), M, K, x.stride(0), xq.data_ptr(), xs.data_ptr(), fmt, block,
                                 _stream(x))
    return xq, xs


def quantize_act_static(x: torch.Tensor, act_scale: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Static scheme: x bf16 [M, K] with one float32 scale (a 1-element CUDA tensor) ->
    (xq float8_e4m3fn [M, K], x_scale [M, ceil(K/128)] float32, all equal to the scale)."""
    _check_bf16_matrix(x, "x")
    if act_scale.dtype != torch.float32 or act_scale.numel() != 1 or act_scale.device != x.device:
        raise ValueError("act_scale must be one float32 on x's device")
    _check_cuda(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    xs = torch.empty((M, _cdiv(K, 128)), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        C.fg8_quantize_act_static(x.data_ptr(), M, K, x.stride(0), act_scale.data_ptr(), xq.data_ptr(), xs.data_ptr(),
                                  _stream(x))
    return xq, xs


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.device != device or not workspace.is_contiguous():
            raise ValueError(f"workspace must be a contiguous tensor on {device}")
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace
    # zero-filled: the first bytes hold the (sticky) device status word
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def linear(x: torch.Tensor, wq: torch.Tensor, w_scale_inv: torch.Tensor, bias: Optional[torch.Tensor] = None,
           scale_fmt="float", out: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, block: int = 128) -> torch.Tensor:
    """y [M, N] bf16 = dequant(quantize_act(x)) . dequant(wq)^T + bias.  block 64
    or 32: 1 x block activation groups and block x block weight blocks, either
    scale format."""
    fmt = scale_fmt_code(scale_fmt)
    _check_bf16_matrix(x, "x")
    M, K = x.shape
    if wq.dim() != 2:
        raise ValueError("wq must be [N, K]")
    N = int(wq.shape[0])
    _check_weight(wq, w_scale_inv, (), N, K, fmt, block, x.device)
    bp = _check_bias(bias, (N,), x.device)
    y = _output(out, M, N, x.device)
    _check_cuda(x, "x")
    nbytes = C.fg8_linear_block_workspace_bytes(M, N, K, fmt, block)  # 0: the call below reports why
    ws = _workspace(nbytes, x.device, workspace)
    with torch.cuda.device(x.device):
        C.fg8_linear_block(x.data_ptr(), M, N, K, x.stride(0), wq.data_ptr(), w_scale_inv.data_ptr(), bp,
                           y.data_ptr(), y.stride(0), fmt, block, ws.data_ptr(), ws.numel() * ws.element_size(),
                           _stream(x))
    return y


def grouped_linear(x: torch.Tensor, row_expert: torch.Tensor, wq: torch.Tensor, w_scale_inv: torch.Tensor,
                   bias: Optional[torch.Tensor] = None, scale_fmt="ue8m0", out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """MoE expert layer over the contiguous grouped layout: x [M, K] bf16 routed
    rows sorted by expert (runs padded to 128-row blocks), row_expert [M]
    int32 (block t uses row_expert[128 t]; -1 skips it), wq [E, N, K],
    w_scale_inv [E, ceil(N/128), ceil(K/128)], bias [E, N] or None.  Rows of
    skipped blocks of the returned y are left as allocated."""
    fmt = scale_fmt_code(scale_fmt)
    _check_bf16_matrix(x, "x")
    M, K = x.shape
    if wq.dim() != 3:
        raise ValueError("wq must be [E, N, K]")
    E, N = int(wq.shape[0]), int(wq.shape[1])
    _check_weight(wq, w_scale_inv, (E,), N, K, fmt, 128, x.device)
    _check_tensor(row_expert, "row_expert", (M,), (torch.int32,), x.device)
    bp = _check_bias(bias, (E, N), x.device)
    y = _output(out, M, N, x.device)
    _check_cuda(x, "x")
    ws = _workspace(C.fg8_grouped_linear_workspace_bytes(M, E, N, K, fmt), x.device, workspace)
    with torch.cuda.device(x.device):
        C.fg8_grouped_linear(x.data_ptr(), M, K, x.stride(0), row_expert.data_ptr(), E, N, wq.data_ptr(),
                             w_scale_inv.data_ptr(), bp, y.data_ptr(), y.stride(0), fmt, ws.data_ptr(),
                             ws.numel() * ws.element_size(), _stream(x))
    return y


def linear_static(x: torch.Tensor, act_scale: torch.Tensor, wq: torch.Tensor, w_scale_inv: torch.Tensor,
                  bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y [M, N] bf16 with x quantized by one precomputed scale (float weight scales)."""
    _check_bf16_matrix(x, "x")
    if act_scale.dtype != torch.float32 or act_scale.numel() != 1 or act_scale.device != x.device:
        raise ValueError("act_scale must be one float32 on x's device")
    M, K = x.shape
    if wq.dim() != 2:
        raise ValueError("wq must be [N, K]")
    N = int(wq.shape[0])
    _check_weight(wq, w_scale_inv, (), N, K, C.FG8_SCALE_FLOAT, 128, x.device)
    bp = _check_bias(bias, (N,), x.device)
    y = _output(out, M, N, x.device)
    _check_cuda(x, "x")
    ws = _workspace(C.fg8_linear_workspace_bytes(M, N, K, C.FG8_SCALE_FLOAT), x.device, workspace)
    with torch.cuda.device(x.device):
        C.fg8_linear_static(x.data_ptr(), M, N, K, x.stride(0), act_scale.data_ptr(), wq.data_ptr(),
                            w_scale_inv.data_ptr(), bp, y.data_ptr(), y.stride(0), ws.data_ptr(),
                            ws.numel() * ws.element_size(), _stream(x))
    return y


def gemm_prequant(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale_inv: torch.Tensor,
                  bias: Optional[torch.Tensor] = None, scale_fmt="float", out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The GEMM on already-quantized activations (layouts of quantize_act)."""
    fmt = scale_fmt_code(scale_fmt)
    if not isinstance(xq, torch.Tensor) or xq.dim() != 2 or wq.dim() != 2:
        raise ValueError("xq must be [M, K] and wq [N, K]")
    M, K = int(xq.shape[0]), int(xq.shape[1])
    N = int(wq.shape[0])
    _check_tensor(xq, "xq", (M, K), _E4M3, xq.device)
    _check_tensor(x_scale, "x_scale", (M, _cdiv(K, 128)), _scale_dtypes(fmt), xq.device)
    _check_weight(wq, w_scale_inv, (), N, K, fmt, 128, xq.device)
    bp = _check_bias(bias, (N,), xq.device)
    y = _output(out, M, N, xq.device)
    _check_cuda(xq, "xq")
    nbytes = C.fg8_gemm_workspace_bytes(M, N, K, fmt)
    ws = _workspace(nbytes, xq.device, workspace)
    with torch.cuda.device(xq.device):
        C.fg8_gemm_prequant(xq.data_ptr(), x_scale.data_ptr(), wq.data_ptr(), w_scale_inv.data_ptr(), bp,
                            y.data_ptr(), M, N, K, y.stride(0), fmt, ws.data_ptr(), ws.numel() * ws.element_size(),
                            _stream(xq))
    return y


def linear_chain(x: torch.Tensor, layers, scale_fmt="float", workspaces=None):
    """Consecutive linears y_i = linear(y_{i-1}, *layers[i]) (layers: [(wq, w_scale_inv, bias or None)]),
    with each layer's activation quantization fused into the previous layer's GEMM epilogue: one
    act-quant launch for the first layer, then one GEMM launch per layer.  Every y_i equals, bit for
    bit, what `linear` gives for that layer on y_{i-1}.  Returns [y_0, ..., y_last]."""
    fmt = scale_fmt_code(scale_fmt)
    _check_bf16_matrix(x, "x")
    layers = list(layers)
    if not layers:
        raise ValueError("layers must hold at least one (wq, w_scale_inv, bias) triple")
    if workspaces is not None and len(workspaces) != len(layers):
        raise ValueError(f"workspaces must hold one entry (a tensor or None) per layer: {len(layers)}")
    M = x.shape[0]
    dims = []
    k = x.shape[1]
    for i, (wq, wsc, b) in enumerate(layers):
        if wq.dim() != 2 or wq.shape[1] != k:
            raise ValueError(f"layer {i}: wq must be [N, {k}]")
        n = int(wq.shape[0])
        try:
            _check_weight(wq, wsc, (), n, k, fmt, 128, x.device)
            _check_bias(b, (n,), x.device)
        except ValueError as e:
            raise ValueError(f"layer {i}: {e}") from None
        dims.append((n, k))
        k = n
    _check_cuda(x, "x")
    if workspaces is None:
        workspaces = [None] * len(layers)
    wss = [_workspace(C.fg8_linear_workspace_bytes(M, n, kk, fmt), x.device, w)
           for (n, kk), w in zip(dims, workspaces)]
    ys = [torch.empty((M, n), dtype=torch.bfloat16, device=x.device) for n, _ in dims]
    s = _stream(x)
    with torch.cuda.device(x.device):
        n0, k0 = dims[0]
        C.fg8_linear_prepare(x.data_ptr(), M, n0, k0, x.stride(0), layers[0][1].data_ptr(), fmt, wss[0].data_ptr(),
                             wss[0].numel(), s)
        for i, ((wq, wsc, b), (n, kk)) in enumerate(zip(layers, dims)):
            bp = 0 if b is None else b.data_ptr()
            if i + 1 < len(layers):
                nn = dims[i + 1][0]
                C.fg8_linear_run_chain(wq.data_ptr(), wsc.data_ptr(), bp, ys[i].data_ptr(), M, n, kk, n, fmt,
                                       wss[i].data_ptr(), wss[i].numel(), nn, layers[i + 1][1].data_ptr(),
                                       wss[i + 1].data_ptr(), wss[i + 1].numel(), s)
            else:
                C.fg8_linear_run(wq.data_ptr(), wsc.data_ptr(), bp, ys[i].data_ptr(), M, n, kk, n, fmt,
                                 wss[i].data_ptr(), wss[i].numel(), s)
    return ys


def dequantize_weight(wq: torch.Tensor, w_scale_inv: torch.Tensor, scale_fmt="float") -> torch.Tensor:
    """Fp8Dequantize: (e4m3 [N, K], block scales) -> bf16 [N, K] with each block's scale folded in."""
    fmt = scale_fmt_code(scale_fmt)
    if not isinstance(wq, torch.Tensor) or wq.dim() != 2:
        raise ValueError("wq must be [N, K]")
    N, K = int(wq.shape[0]), int(wq.shape[1])
    _check_weight(wq, w_scale_inv, (), N, K, fmt, 128, wq.device)
    _check_cuda(wq, "wq")
    w = torch.empty((N, K), dtype=torch.bfloat16, device=wq.device)
    with torch.cuda.device(wq.device):
        C.fg8_dequantize_weight(wq.data_ptr(), N, K, w_scale_inv.data_ptr(), fmt, w.data_ptr(), K, _stream(wq))
    return w


def scale_to_ue8m0(scale: torch.Tensor) -> Tuple[torch.Tensor, int]:
    """float32 power-of-two scales (a checkpoint's ".scale" key) -> (float8_e8m0fnu scales of the same
    shape, number of inputs that were no UE8M0 value; those become NaN).  Synchronizes for the count."""
    s = scale.contiguous()
    if s.dtype != torch.float32 or not s.is_cuda:
        raise ValueError("scale must be a float32 CUDA tensor")
    out = torch.empty(s.shape, dtype=torch.uint8, device=s.device)
    bad = torch.zeros(1, dtype=torch.int32, device=s.device)
    with torch.cuda.device(s.device):
        C.fg8_scale_to_ue8m0(s.data_ptr(), s.numel(), out.data_ptr(), bad.data_ptr(), _stream(s))
    return out.view(torch.float8_e8m0fnu), int(bad.item())


class FP8Linear(torch.nn.Module):
    """Inference linear layer holding a quantized weight ([zh] §一 FP8Linear):
    weight float8_e4m3fn [out, in], weight_scale_inv per block x block block
    (weight_block_size (128, 128) by default, or (64, 64) or (32, 32)),
    bias kept in bf16 (not quantized, [zh] §三).  The layer keeps one device
    workspace, so forwards of the same layer on different CUDA streams must
    not overlap in time (use one layer object per concurrent stream)."""

    def __init__(self, weight: torch.Tensor, bias: Optional[torch.Tensor] = None, scale_fmt="float",
                 block: int = 128):
        """Quantizes `weight` (bf16 [out, in], or any float dtype, cast to bf16) on its device."""
        super().__init__()
        fmt = scale_fmt_code(scale_fmt)
        wq, ws = quantize_weight(weight.to(torch.bfloat16).contiguous(), fmt, block)
        self._hold(wq, ws, bias, fmt, block)

    @classmethod
    def from_quantized(cls, weight: torch.Tensor, weight_scale_inv: torch.Tensor,
                       bias: Optional[torch.Tensor] = None, scale_fmt="float", block: int = 128) -> "FP8Linear":
        """The layer over a weight that is already quantized, as a pre-quantized
        checkpoint stores it ([zh] §五): `weight` e4m3 [out, in] and
        `weight_scale_inv` [ceil(out/block), ceil(in/block)], float32, or UE8M0
        for scale_fmt "ue8m0" (a checkpoint's float32 power-of-two scales
        convert exactly with scale_to_ue8m0).  Raw uint8 bytes are taken as
        those dtypes.  No kernel runs; the tensors are kept, not copied."""
        fmt = scale_fmt_code(scale_fmt)
        if not isinstance(weight, torch.Tensor) or weight.dim() != 2:
            raise ValueError("weight must be [out, in]")
        N, K = int(weight.shape[0]), int(weight.shape[1])
        _check_weight(weight, weight_scale_inv, (), N, K, fmt, block, weight.device)
        if bias is not None:
            bias = bias.to(torch.bfloat16).contiguous()
            _check_bias(bias, (N,), weight.device)
        layer = cls.__new__(cls)
        torch.nn.Module.__init__(layer)
        layer._hold(weight.view(torch.float8_e4m3fn), weight_scale_inv.view(_SCALE_DTYPES[fmt]), bias, fmt, block)
        return layer

    def _hold(self, wq, ws, bias, fmt, block):
        self.scale_fmt = fmt
        self.block = block
        self.register_buffer("weight", wq)
        self.register_buffer("weight_scale_inv", ws)
        self.register_buffer("bias", None if bias is None else bias.to(torch.bfloat16).contiguous())
        self._ws = None

    @property
    def in_features(self) -> int:
        return self.weight.shape[1]

    @property
    def out_features(self) -> int:
        return self.weight.shape[0]

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, x.shape[-1]).to(torch.bfloat16).contiguous()
        M, N, K = x2.shape[0], self.out_features, self.in_features
        need = C.fg8_linear_block_workspace_bytes(M, N, K, self.scale_fmt, self.block)
        if self._ws is None or self._ws.numel() < need or self._ws.device != x2.device:
            self._ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=x2.device)
        y = linear(x2, self.weight, self.weight_scale_inv, self.bias, self.scale_fmt, workspace=self._ws,
                   block=self.block)
        return y.reshape(*lead, N)
