"""Seeded synthetic inputs shaped like the pages' models.

This module only draws random tensors; it holds none of the quantization or
GEMM arithmetic, so both the CUDA library's tests and the CPU oracle can take
their inputs from it without sharing any of the method.

Shapes come from the models the pages name: ESM-2 35M (hidden 480, FFN 1920,
max length 1022), Llama-3-8B projections (4096 <-> 14336) and DeepSeek-V3
dense MLP projections (7168 <-> 18432), plus a square 12288 sweep.  No dataset
or checkpoint is used; every tensor is drawn from a seeded torch generator in
float32 and rounded once to bf16 (round-to-nearest-even).

Seed plan: config i uses base seed i-1; offsets +0 for x, +1 for W (or W1),
+2 for W2, +3 for bias, +4 for outlier / per-row magnitude draws.
"""
import dataclasses
import math
from typing import Optional, Tuple

import torch

FMT_FLOAT = 0
FMT_UE8M0 = 1


@dataclasses.dataclass(frozen=True)
class Gemm:
    """One linear layer y[M,N] = x[M,K] . W[N,K]^T + bias[N]."""
    name: str
    M: int
    K: int
    N: int
    fmt: int


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """float32 N(0, std^2) from a seeded generator, rounded once to bf16."""
    g = _gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def x_normal(M: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    return normal((M, K), 1.0, seed, device)


def x_outliers(M: int, K: int, seed: int, device="cpu", frac: float = 0.01, factor: float = 20.0) -> torch.Tensor:
    """x ~ N(0,1) with round(frac*K) channels (a seeded permutation) scaled by factor."""
    g = _gen(seed, device)
    t = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    go = _gen(seed + 4, "cpu")
    n_out = int(round(frac * K))
    cols = torch.randperm(K, generator=go)[:n_out].to(device)
    t[:, cols] *= factor
    return t.to(torch.bfloat16)


def x_student_t(M: int, K: int, seed: int, device="cpu", nu: int = 4, clip: float = 50.0) -> torch.Tensor:
    """Student-t(nu) drawn as z / sqrt(chi2_nu / nu), chi2 as a sum of nu squared normals; clipped."""
    g = _gen(seed, device)
    z = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(M, K, device=device, dtype=torch.float32)
    for _ in range(nu):
        u = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
        chi2.addcmul_(u, u)
    t = z / torch.sqrt(chi2 / nu)
    return t.clamp_(-clip, clip).to(torch.bfloat16)


def w_row_groups(N: int, K: int, std: float, seed: int, device="cpu", lo: float = 0.25, hi: float = 4.0,
                 rows_per_group: int = 128) -> torch.Tensor:
    """W ~ N(0, std^2) times g_r = exp(U(ln lo, ln hi)), one g per 128-row group of N."""
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
    go = _gen(seed + 4, "cpu")
    n_groups = (N + rows_per_group - 1) // rows_per_group
    u = torch.rand(n_groups, generator=go, dtype=torch.float64)
    mag = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).to(torch.float32)
    mag = mag.repeat_interleave(rows_per_group)[:N].to(device)
    w.mul_(std).mul_(mag[:, None])
    return w.to(torch.bfloat16)


# ------------------------------------------------------------------ configs --
TINY = Gemm("tiny", 16, 256, 256, FMT_FLOAT)
ESM_W1 = Gemm("esm2_w1", 8 * 1022, 480, 1920, FMT_FLOAT)
ESM_W2 = Gemm("esm2_w2", 8 * 1022, 1920, 480, FMT_FLOAT)
LLAMA_M = (1, 16, 128, 4096)
DSV3_UP = Gemm("dsv3_up", 8192, 7168, 18432, FMT_UE8M0)
DSV3_DOWN = Gemm("dsv3_down", 8192, 18432, 7168, FMT_UE8M0)
SQUARE_M = (1, 8, 64, 512, 2048, 8192, 16384)


def llama(M: int, which: str) -> Gemm:
    if which == "gate_up":
        return Gemm(f"llama_gate_up_m{M}", M, 4096, 14336, FMT_FLOAT)
    return Gemm(f"llama_down_m{M}", M, 14336, 4096, FMT_FLOAT)


def square(M: int, fmt: int) -> Gemm:
    return Gemm(f"square_m{M}_{'ue8m0' if fmt else 'float'}", M, 12288, 12288, fmt)


def make_inputs(cfg: str, gemm: Gemm, device="cpu", stage: int = 1) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(x bf16 [M,K], W bf16 [N,K], bias bf16 [N]) for one layer of a config.

    cfg is one of "tiny", "esm2", "llama", "dsv3", "square"; stage 1 or 2
    selects W1/W2 (esm2: the two FFN matrices; llama: gate/up then down;
    dsv3: up then down).
    """
    base = {"tiny": 0, "esm2": 1, "llama": 2, "dsv3": 3, "square": 4}[cfg]
    M, K, N = gemm.M, gemm.K, gemm.N
    w_seed = base + (1 if stage == 1 else 2)
    if cfg == "llama":
        x = x_outliers(M, K, base, device)
    elif cfg == "dsv3":
        x = x_student_t(M, K, base, device)
    else:
        x = x_normal(M, K, base, device)
    if cfg == "dsv3":
        w = w_row_groups(N, K, 0.015, w_seed, device)
    elif cfg == "square":
        w = normal((N, K), 0.01, w_seed, device)
    else:
        w = normal((N, K), 0.02, w_seed, device)
    bias = normal((N,), 0.1, base + 3 + (10 if stage == 2 else 0), device)
    return x, w, bias


# ----------------------------------------------------- MoE experts ----
# DeepSeek-V3-shaped routed experts (hidden 7168, expert intermediate 2048,
# 256 experts, 8 per token); the expert kernels take UE8M0 scales on
# Blackwell.  gate/up: K = 7168 -> N = 2 x 2048; down: K = 2048 -> N = 7168.
MOE_BLOCK = 128
DSV3_MOE = dict(experts=256, topk=8, hidden=7168, inter=2048, tokens=4096, skew=0.5)


def moe_routing(T: int, E: int, topk: int, seed: int, skew: float = 1.0):
    """Seeded synthetic routing in the contiguous grouped layout.

    Expert popularity is log-normal (sigma = skew); each token picks topk
    distinct experts with probability proportional to popularity (Gumbel
    top-k).  The T * topk routed rows are sorted by expert (then token) and
    each expert's run is padded with rows of token -1 to a whole number of
    MOE_BLOCK-row blocks.  Returns (row_token, row_expert) int64 / int32
    tensors of the padded length: row_expert is -1 on padding rows.
    """
    g = _gen(seed, "cpu")
    logp = torch.randn(E, generator=g, dtype=torch.float64) * skew
    gumbel = -torch.log(-torch.log(torch.rand(T, E, generator=g, dtype=torch.float64).clamp_min(1e-300)))
    picks = torch.topk(logp[None, :] + gumbel, topk, dim=1).indices  # [T, topk], distinct per token
    tok = torch.arange(T).repeat_interleave(topk)
    exp = picks.reshape(-1)
    order = torch.argsort(exp * T + tok)
    tok, exp = tok[order], exp[order]
    counts = torch.bincount(exp, minlength=E)
    padded = (counts + MOE_BLOCK - 1) // MOE_BLOCK * MOE_BLOCK
    Mp = int(padded.sum())
    row_token = torch.full((Mp,), -1, dtype=torch.int64)
    row_expert = torch.full((Mp,), -1, dtype=torch.int32)
    starts = torch.cumsum(padded, 0) - padded
    src = 0
    for e in range(E):
        n = int(counts[e])
        if n:
            a = int(starts[e])
            row_token[a:a + n] = tok[src:src + n]
            row_expert[a:a + n] = e
            src += n
    return row_token, row_expert


def gather_rows(x: torch.Tensor, row_token: torch.Tensor) -> torch.Tensor:
    """x[row_token] with zero rows where row_token is -1."""
    out = torch.zeros(row_token.numel(), x.shape[1], dtype=x.dtype, device=x.device)
    keep = row_token >= 0
    out[keep.to(x.device)] = x[row_token[keep].to(x.device)]
    return out


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")


def from_bits(a, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
