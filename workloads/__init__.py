"""Seeded synthetic inputs for the fine-grained FP8 W8A8 workloads.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic (no amax, scale, rounding or GEMM), so both the CPU oracle
and the CUDA library can be fed from it.

Recipe (every tensor drawn in fp32 with a seeded ``torch.Generator`` on the
requested device, then rounded to bf16 round-to-nearest-even):
  * activations ~ N(0, 1); with ``outliers`` each element is independently
    multiplied by 50 with probability 0.001;
  * the down-projection input is sign(z) * |z|^1.5 with z ~ N(0, 1) (a
    post-SiLU-like heavy tail);
  * weights ~ N(0, 0.02) (0.02 is the standard deviation);
  * seeds: X uses ``seed``, W uses ``seed + 1``, MoE routing ``seed + 2``; MoE
    expert e's weights use their own generator seeded ``(seed + 1) * 4096 + e``
    so that any expert can be regenerated alone.
The shapes stand in for Llama-3-8B and DeepSeek-V3 layers; no model weights
or datasets are involved.  CPU and CUDA generators give different streams, so
a test always feeds the oracle the same bytes the GPU saw.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

SCALE_F32 = 0
SCALE_UE8M0 = 1


@dataclass(frozen=True)
class Linear:
    """One dense W8A8 linear layer: X [M, K] x W [N, K]^T."""
    name: str
    M: int
    N: int
    K: int
    fmt: int
    x_kind: str = "normal_outliers"   # "normal", "normal_outliers", "heavy_tail"
    seed: int = 0


@dataclass(frozen=True)
class MoE:
    """M-grouped expert layer: tokens routed top-k to E experts."""
    name: str
    E: int = 256
    N: int = 4096
    K: int = 7168
    tokens: int = 4096
    topk: int = 8
    zipf: float = 1.1
    fmt: int = SCALE_UE8M0
    seed: int = 0


TINY = Linear("tiny_128x256x512", 128, 256, 512, SCALE_F32)
LLAMA_ATTN = Linear("llama3_8b_attn_proj_4096x4096x4096", 4096, 4096, 4096, SCALE_F32)
LLAMA_GATE_UP = Linear("llama3_8b_gate_up_8192x28672x4096", 8192, 28672, 4096, SCALE_F32)
LLAMA_DOWN = Linear("llama3_8b_down_8192x4096x14336", 8192, 4096, 14336, SCALE_F32,
                    x_kind="heavy_tail")
DS_DECODE = {m: Linear(f"deepseek_v3_decode_m{m}_18432x7168", m, 18432, 7168, SCALE_UE8M0,
                       x_kind="normal") for m in (1, 8, 32, 64)}
MOE = MoE("deepseek_v3_moe_256x4096x7168_top8")
# the same expert shapes with 32 experts and 512 tokens (~1 GB of weights): a
# profiling case larger than L2 but small enough for multi-pass captures
MOE_SMALL = MoE("deepseek_v3_moe_32x4096x7168_top8_512tok", E=32, tokens=512)
# the expert layer with fp32 block scales (the promotion kernel's grouped path)
MOE_F32 = replace(MOE, name="deepseek_v3_moe_256x4096x7168_top8_fp32", fmt=SCALE_F32)
# decode step of the same expert layer: 128 tokens, top-8, in the masked
# layout (every expert a fixed block of 128 rows, its first counts[e] used)
MOE_DECODE = MoE("deepseek_v3_moe_decode_masked_256x4096x7168_top8_128tok", tokens=128)
MOE_DECODE_SMALL = MoE("deepseek_v3_moe_decode_masked_32x4096x7168_top8_64tok", E=32, tokens=64)

# the dense prefill shapes with power-of-two (UE8M0) scales: the tensor core's
# block-scaled MMA path instead of the fp32 promotion
LLAMA_UE8M0 = {c.name: replace(c, name=f"{c.name}_ue8m0", fmt=SCALE_UE8M0)
               for c in (LLAMA_ATTN, LLAMA_GATE_UP, LLAMA_DOWN)}
LINEARS = {c.name: c for c in [TINY, LLAMA_ATTN, LLAMA_GATE_UP, LLAMA_DOWN, *DS_DECODE.values(),
                               *LLAMA_UE8M0.values()]}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(shape, kind: str, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if kind == "normal_outliers":
        u = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
        z = torch.where(u < 0.001, z * 50.0, z)
    elif kind == "heavy_tail":
        z = torch.sign(z) * z.abs().pow(1.5)
    elif kind != "normal":
        raise ValueError(kind)
    return z.to(torch.bfloat16)


def weights(shape, seed: int, device="cpu", std: float = 0.02) -> torch.Tensor:
    g = _gen(device, seed)
    w = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def linear_inputs(cfg: Linear, device="cpu"):
    """(X bf16 [M, K], W bf16 [N, K]) for a dense layer."""
    X = activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device)
    W = weights((cfg.N, cfg.K), cfg.seed + 1, device)
    return X, W


def scaled_linear(cfg: Linear, M=None, N=None, K=None, **kw) -> Linear:
    """The same recipe at another shape (for parity tests that must finish on
    the CPU oracle in seconds)."""
    from dataclasses import replace
    return replace(cfg, name=f"{cfg.name}@{M or cfg.M}x{N or cfg.N}x{K or cfg.K}",
                   M=M or cfg.M, N=N or cfg.N, K=K or cfg.K, **kw)


# ----------------------------------------------------------------- MoE
@dataclass
class Routing:
    counts: np.ndarray          # int64 [E] real rows per expert
    group_offs: np.ndarray      # int32 [E+1] padded segment starts (multiples of 128)
    row_token: np.ndarray       # int64 [M_total] source token of each row, -1 = padding
    M_total: int = field(default=0)


def moe_routing(cfg: MoE, pad: int = 128) -> Routing:
    """Top-k routing with Zipf-skewed expert popularity: p(expert r-1) is
    proportional to 1/r^zipf; each token draws topk distinct experts by
    Gumbel-top-k on log p.  Rows are grouped per expert in expert order
    (tokens ascending inside a segment) and each segment is zero-padded to a
    multiple of ``pad`` rows."""
    g = _gen("cpu", cfg.seed + 2)
    ranks = torch.arange(1, cfg.E + 1, dtype=torch.float64)
    logp = -cfg.zipf * torch.log(ranks)
    logp = logp - torch.logsumexp(logp, 0)
    u = torch.rand((cfg.tokens, cfg.E), generator=g, dtype=torch.float64)
    u = u.clamp_min(1e-300)
    gumbel = -torch.log(-torch.log(u))
    top = torch.topk(logp[None, :] + gumbel, cfg.topk, dim=1).indices.numpy()
    counts = np.bincount(top.reshape(-1), minlength=cfg.E).astype(np.int64)
    seg = (counts + pad - 1) // pad * pad
    offs = np.zeros(cfg.E + 1, dtype=np.int64)
    offs[1:] = np.cumsum(seg)
    M_total = int(offs[-1])
    row_token = np.full(M_total, -1, dtype=np.int64)
    fill = offs[:-1].copy()
    for t in range(cfg.tokens):            # tokens ascending inside each segment
        for e in sorted(top[t]):
            row_token[fill[e]] = t
            fill[e] += 1
    return Routing(counts, offs.astype(np.int32), row_token, M_total)


def moe_tokens(cfg: MoE, device="cpu") -> torch.Tensor:
    """Token activations X_tok bf16 [tokens, K] ~ N(0, 1)."""
    return activations((cfg.tokens, cfg.K), "normal", cfg.seed, device)


def moe_grouped_rows(X_tok: torch.Tensor, routing: Routing) -> torch.Tensor:
    """X [M_total, K]: row i is X_tok[row_token[i]] (duplicated per routed
    expert) or zeros for padding rows."""
    idx = torch.as_tensor(routing.row_token, device=X_tok.device)
    X = torch.zeros((routing.M_total, X_tok.shape[1]), dtype=X_tok.dtype, device=X_tok.device)
    valid = idx >= 0
    X[valid] = X_tok[idx[valid]]
    return X


def moe_masked_rows(X_tok: torch.Tensor, routing: Routing, E: int, cap: int) -> torch.Tensor:
    """X [E * cap, K] in the masked layout: expert e's routed tokens (in
    ascending token order) in rows [e * cap, e * cap + counts[e]), zeros in
    the rest of its block."""
    X = torch.zeros((E * cap, X_tok.shape[1]), dtype=X_tok.dtype, device=X_tok.device)
    for e in range(E):
        seg = routing.row_token[routing.group_offs[e]:routing.group_offs[e] + routing.counts[e]]
        if len(seg):
            X[e * cap:e * cap + len(seg)] = X_tok[torch.as_tensor(seg, device=X_tok.device)]
    return X


def moe_expert_weight(cfg: MoE, e: int, device="cpu") -> torch.Tensor:
    """Expert e's bf16 weight [N, K] ~ N(0, 0.02), regenerable alone."""
    return weights((cfg.N, cfg.K), (cfg.seed + 1) * 4096 + e, device)


def scaled_moe(cfg: MoE, **kw) -> MoE:
    from dataclasses import replace
    return replace(cfg, name=cfg.name + "@" + ",".join(f"{k}={v}" for k, v in kw.items()), **kw)
