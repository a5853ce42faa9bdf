"""The Python binding's operand checks, on CPU.

The C ABI takes raw pointers, so a scale tensor of the wrong shape or dtype
would be read out of bounds by a kernel.  The wrappers check every operand
against the shape, dtype and device the call implies before passing a
pointer on; these tests feed each wrapper one wrong operand at a time and
expect a ValueError naming it.  With every operand right but on the CPU the
last check (CUDA device) fires, so no CPU pointer ever reaches the library.
"""
import pytest
import torch

import fine_grained_fp8_act_b200 as fg8

BF16, F32, U8 = torch.bfloat16, torch.float32, torch.uint8
E4M3, E8M0 = torch.float8_e4m3fn, torch.float8_e8m0fnu
M, N, K = 40, 264, 400          # ragged against 128 and 32
Nb, Kb = 3, 4                   # ceil(264 / 128), ceil(400 / 128)


def _dense(fmt="float", block=128):
    nb, kb = -(-N // block), -(-K // block)
    x = torch.zeros(M, K, dtype=BF16)
    wq = torch.zeros(N, K, dtype=E4M3)
    ws = torch.zeros(nb, kb, dtype=F32 if fmt == "float" else E8M0)
    b = torch.zeros(N, dtype=BF16)
    return x, wq, ws, b


def _raises(match, fn, *a, **k):
    with pytest.raises(ValueError, match=match):
        fn(*a, **k)


@pytest.mark.parametrize("fmt", ["float", "ue8m0"])
def test_linear_operands(fmt):
    x, wq, ws, b = _dense(fmt)
    _raises("must be a CUDA tensor", fg8.linear, x, wq, ws, b, fmt)
    _raises("wq must be", fg8.linear, x, wq.to(BF16), ws, b, fmt)
    _raises("wq must have shape", fg8.linear, x, wq[:, :K - 16].contiguous(), ws, b, fmt)
    _raises("wq must be contiguous", fg8.linear, x, torch.zeros(K, N, dtype=E4M3).t(), ws, b, fmt)
    _raises("w_scale_inv must have shape", fg8.linear, x, wq, ws[:, :Kb - 1].contiguous(), b, fmt)
    _raises("w_scale_inv must have shape", fg8.linear, x, wq, ws.t().contiguous(), b, fmt)
    other = torch.zeros(Nb, Kb, dtype=E8M0 if fmt == "float" else F32)
    _raises("w_scale_inv must be", fg8.linear, x, wq, other, b, fmt)
    _raises("bias must have shape", fg8.linear, x, wq, ws, b[:N - 1].contiguous(), fmt)
    _raises("bias must be", fg8.linear, x, wq, ws, b.float(), fmt)
    _raises("out must be", fg8.linear, x, wq, ws, b, fmt, out=torch.empty(M, N + 1, dtype=BF16)[:, :N - 1])
    _raises("out must have unit stride", fg8.linear, x, wq, ws, b, fmt, out=torch.empty(N, M, dtype=BF16).t())
    _raises("x must be a 2-D bf16", fg8.linear, x.float(), wq, ws, b, fmt)
    _raises("x must have unit stride", fg8.linear, x.as_strided((M, K), (K // 2, 1)), wq, ws, b, fmt)
    # raw bytes are the same bits: accepted (up to the device check)
    wsb = ws.view(U8) if fmt == "ue8m0" else ws
    _raises("must be a CUDA tensor", fg8.linear, x, wq.view(U8), wsb, None, fmt)
    # row-strided x and out are fine
    xs = torch.zeros(M, K + 64, dtype=BF16)[:, :K]
    _raises("must be a CUDA tensor", fg8.linear, xs, wq, ws, b, fmt, out=torch.empty(M, N + 8, dtype=BF16)[:, :N])


def test_linear_block32_operands():
    x, wq, ws, b = _dense("ue8m0", block=32)
    assert ws.shape == (9, 13)
    _raises("must be a CUDA tensor", fg8.linear, x, wq, ws, b, "ue8m0", block=32)
    _raises("w_scale_inv must have shape", fg8.linear, x, wq, ws, b, "ue8m0", block=128)
    _, _, ws128, _ = _dense("ue8m0")
    _raises("w_scale_inv must have shape", fg8.linear, x, wq, ws128, b, "ue8m0", block=32)


def test_grouped_linear_operands():
    E = 3
    x = torch.zeros(256, K, dtype=BF16)
    re = torch.zeros(256, dtype=torch.int32)
    wq = torch.zeros(E, N, K, dtype=E4M3)
    ws = torch.zeros(E, Nb, Kb, dtype=E8M0)
    b = torch.zeros(E, N, dtype=BF16)
    _raises("must be a CUDA tensor", fg8.grouped_linear, x, re, wq, ws, b)
    _raises("wq must be", fg8.grouped_linear, x, re, wq[0], ws, b)
    _raises("w_scale_inv must have shape", fg8.grouped_linear, x, re, wq, ws[:E - 1].contiguous(), b)
    _raises("w_scale_inv must be", fg8.grouped_linear, x, re, wq, ws.float(), b)
    _raises("row_expert must be", fg8.grouped_linear, x, re.long(), wq, ws, b)
    _raises("row_expert must have shape", fg8.grouped_linear, x, re[:255].contiguous(), wq, ws, b)
    _raises("bias must have shape", fg8.grouped_linear, x, re, wq, ws, b[0].contiguous())
    _raises("must be a CUDA tensor", fg8.grouped_linear, x, re, wq, ws.view(U8), None)


def test_static_prequant_chain_dequant_operands():
    x, wq, ws, b = _dense("float")
    s = torch.ones(1, dtype=F32)
    _raises("must be a CUDA tensor", fg8.linear_static, x, s, wq, ws, b)
    _raises("w_scale_inv must be", fg8.linear_static, x, s, wq, ws.to(E8M0), b)
    _raises("wq must have shape", fg8.linear_static, x, s, torch.zeros(N, K + 16, dtype=E4M3), ws, b)

    xq = torch.zeros(M, K, dtype=E4M3)
    xs = torch.zeros(M, Kb, dtype=F32)
    _raises("must be a CUDA tensor", fg8.gemm_prequant, xq, xs, wq, ws, b, "float")
    _raises("x_scale must have shape", fg8.gemm_prequant, xq, xs.t().contiguous(), wq, ws, b, "float")
    _raises("x_scale must be", fg8.gemm_prequant, xq, xs.to(E8M0), wq, ws, b, "float")
    _raises("xq must be", fg8.gemm_prequant, xq.to(BF16), xs, wq, ws, b, "float")

    wq2 = torch.zeros(K, N, dtype=E4M3)
    ws2 = torch.zeros(Kb, Nb, dtype=F32)
    _raises("must be a CUDA tensor", fg8.linear_chain, x, [(wq, ws, b), (wq2, ws2, None)])
    _raises("layer 1: w_scale_inv must have shape", fg8.linear_chain, x, [(wq, ws, b), (wq2, ws, None)])
    _raises("layer 1: wq must be", fg8.linear_chain, x, [(wq, ws, b), (wq, ws, None)])
    _raises("at least one", fg8.linear_chain, x, [])
    _raises("one entry", fg8.linear_chain, x, [(wq, ws, b), (wq2, ws2, None)], workspaces=[None])

    _raises("must be a CUDA tensor", fg8.dequantize_weight, wq, ws, "float")
    _raises("w_scale_inv must have shape", fg8.dequantize_weight, wq, ws[:1].contiguous(), "float")


@pytest.mark.parametrize("fmt,block", [("float", 128), ("ue8m0", 128), ("ue8m0", 32)])
def test_fp8linear_from_quantized(fmt, block):
    """A layer over a pre-quantized checkpoint's tensors: kept as given (raw
    bytes viewed as float8), checked against the block shape rule, and its
    forward refuses CPU tensors instead of computing on the host."""
    _, wq, ws, b = _dense(fmt, block)
    layer = fg8.FP8Linear.from_quantized(wq, ws, b, fmt, block=block)
    assert (layer.in_features, layer.out_features, layer.block) == (K, N, block)
    assert layer.weight.data_ptr() == wq.data_ptr() and layer.weight_scale_inv.data_ptr() == ws.data_ptr()
    assert set(layer.state_dict()) == {"weight", "weight_scale_inv", "bias"}
    raw = fg8.FP8Linear.from_quantized(wq.view(U8), ws.view(U8) if fmt == "ue8m0" else ws, None, fmt, block=block)
    assert raw.weight.dtype == E4M3 and raw.weight_scale_inv.dtype == (F32 if fmt == "float" else E8M0)
    assert raw.bias is None
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        layer(torch.zeros(2, 3, K, dtype=BF16))
    other = 128 if block == 32 else 32
    _raises("w_scale_inv must have shape", fg8.FP8Linear.from_quantized, wq, ws, b, fmt, block=other)
    _raises("bias must have shape", fg8.FP8Linear.from_quantized, wq, ws, b[:N - 8], fmt, block=block)
    _raises("weight must be", fg8.FP8Linear.from_quantized, wq[0], ws, b, fmt, block=block)
    # a state dict moves between layers built this way
    twin = fg8.FP8Linear.from_quantized(torch.ones_like(wq), torch.ones_like(ws), torch.ones_like(b), fmt, block)
    twin.load_state_dict(layer.state_dict())
    assert torch.equal(twin.weight.view(U8), wq.view(U8)) and torch.equal(twin.bias, b)


@pytest.mark.parametrize("fmt,block", [("float", 128), ("ue8m0", 32)])
def test_fp8linear_init_holds_what_quantize_weight_returns(monkeypatch, orc, fmt, block):
    """FP8Linear(weight) keeps quantize_weight's outputs as its buffers (the
    device quantizer replaced by the oracle here, so this runs on CPU)."""
    from fine_grained_fp8_act_b200 import layer as L
    code = 0 if fmt == "float" else 1

    def on_host(w, f, b):
        assert (f, b) == (code, block) and w.dtype == BF16 and w.is_contiguous()
        q, s = orc.quantize_weight(w.view(torch.int16).numpy().view("uint16"), f, b)
        s = torch.from_numpy(s)
        return torch.from_numpy(q).view(E4M3), (s if f == 0 else s.view(E8M0))
    monkeypatch.setattr(L, "quantize_weight", on_host)
    w = torch.randn(N, K).mul(0.02)                       # float32: cast to bf16 by the layer
    b = torch.randn(N)
    layer = fg8.FP8Linear(w, b, fmt, block=block)
    q, s = on_host(w.to(BF16).contiguous(), code, block)
    assert torch.equal(layer.weight.view(U8), q.view(U8)) and torch.equal(layer.weight_scale_inv.view(U8), s.view(U8))
    assert layer.bias.dtype == BF16 and torch.equal(layer.bias, b.to(BF16))
    assert (layer.scale_fmt, layer.block, layer.in_features, layer.out_features) == (code, block, K, N)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        layer(torch.zeros(5, K, dtype=BF16))
