"""Seeded synthetic inputs for the W4A4 / MXFP4 linear layer workloads.

This module only draws random tensors (shapes, distributions, outlier channels, MoE routing); it
holds none of the method's arithmetic, and both the CUDA path and the CPU oracle receive exactly
the tensors it returns (bf16 bits for X and W, fp32 for s).

Recipe (every workload):
  * one ``torch.Generator('cpu')`` per case, seed = 1000 * workload + sweep index;
  * draw order: s, outlier channel set, X, W;
  * s[k] = exp(U(ln 0.5, ln 8)), fp32 (log-uniform on [0.5, 8]);
  * outlier channels: a seeded choice without replacement; those X columns are multiplied by the
    workload's factor;
  * X and W are drawn in fp32 and rounded to bf16 (round-to-nearest-even, torch's cast).

device="cuda" draws the same recipe with a CUDA generator (same shapes and distributions, other
bits): the benchmark uses it for the large workloads; the parity tests always draw on the CPU.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

LN_LO, LN_HI = math.log(0.5), math.log(8.0)


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device)
    g.manual_seed(int(seed))
    return g


def log_uniform_scale(g: torch.Generator, K: int) -> torch.Tensor:
    u = torch.rand(K, generator=g, dtype=torch.float64, device=g.device)
    return torch.exp(LN_LO + (LN_HI - LN_LO) * u).to(torch.float32)


def outlier_channels(g: torch.Generator, K: int, count: int) -> torch.Tensor:
    return torch.randperm(K, generator=g, device=g.device)[:count].sort().values


def normal_bf16(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return (torch.randn(*shape, generator=g, dtype=torch.float32, device=g.device) * std).to(torch.bfloat16)


@dataclass
class DenseCase:
    """One dense linear: X [M, K] bf16, W [N, K] bf16, s [K] fp32."""
    name: str
    X: torch.Tensor
    W: torch.Tensor
    s: torch.Tensor
    had_block: int
    outliers: torch.Tensor


def dense_case(seed: int, M: int, K: int, N: int, *, w_std: float = 0.02, n_outliers: int = 0,
               outlier_factor: float = 1.0, heavy_tail: bool = False, had_block: int = 32,
               name: str = "dense", draw_w: bool = True, device: str = "cpu") -> DenseCase:
    """X ~ N(0, 1) (or sigma_k * N(0, 1) with sigma_k = |t_3| per channel when heavy_tail), with the
    outlier channels scaled by outlier_factor; W ~ N(0, w_std); s log-uniform [0.5, 8]."""
    g = _gen(seed, device)
    s = log_uniform_scale(g, K)
    out = outlier_channels(g, K, n_outliers)
    if heavy_tail:
        # Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3)
        z = torch.randn(K, generator=g, dtype=torch.float64, device=g.device)
        chi2 = (torch.randn(3, K, generator=g, dtype=torch.float64, device=g.device) ** 2).sum(0)
        sigma = (z / torch.sqrt(chi2 / 3.0)).abs().to(torch.float32)
    else:
        sigma = torch.ones(K, dtype=torch.float32, device=g.device)
    if n_outliers:
        sigma = sigma.clone()
        sigma[out] *= outlier_factor
    X = (torch.randn(M, K, generator=g, dtype=torch.float32, device=g.device) * sigma).to(torch.bfloat16)
    W = normal_bf16(g, (N, K), w_std) if draw_w else None
    return DenseCase(name, X, W, s, had_block, out)


# ----------------------------------------------------------------------------------------------
# The five workloads. Sizes follow the workload list of the project; each function documents it.
# ----------------------------------------------------------------------------------------------

def tiny(had_block: int = 32, sweep: int = 0) -> DenseCase:
    """Tiny dense linear: X [16, 256] ~ N(0,1), 4 outlier channels x50; W [256, 256] ~ N(0, 0.02)."""
    return dense_case(1000 * 1 + sweep, 16, 256, 256, w_std=0.02, n_outliers=4, outlier_factor=50.0,
                      had_block=had_block, name="tiny_16x256x256")


LLAMA3_8B_UP = dict(K=4096, N=14336)
LLAMA3_8B_M = (1, 16, 128, 2048)


def llama3_8b_up(M: int, had_block: int = 32, sweep: int | None = None, draw_w: bool = True) -> DenseCase:
    """Llama-3-8B-shaped MLP up/gate projection: K=4096, N=14336; 0.5% outlier channels x30."""
    K, N = LLAMA3_8B_UP["K"], LLAMA3_8B_UP["N"]
    idx = LLAMA3_8B_M.index(M) if (sweep is None and M in LLAMA3_8B_M) else (sweep or 0)
    return dense_case(1000 * 2 + idx, M, K, N, w_std=0.02, n_outliers=round(0.005 * K), outlier_factor=30.0,
                      had_block=had_block, name=f"llama3_8b_up_M{M}_b{had_block}", draw_w=draw_w)


QWEN3_32B_LINEARS = (  # (name, K, N, input id): q/k/v share one input, gate/up share one
    ("q_proj", 5120, 8192, "qkv"), ("k_proj", 5120, 1024, "qkv"), ("v_proj", 5120, 1024, "qkv"),
    ("o_proj", 8192, 5120, "o"), ("gate_proj", 5120, 25600, "gateup"), ("up_proj", 5120, 25600, "gateup"),
    ("down_proj", 25600, 5120, "down"),
)
QWEN3_32B_M = (1, 8, 64, 4096)


def qwen3_32b_layer(M: int, sweep: int = 0, draw_w: bool = True, device: str = "cpu"):
    """Qwen3-32B-shaped decoder-layer linears. Each distinct input (qkv, o, gateup, down) gets its own
    X (heavy-tailed channel magnitudes) and s; W ~ N(0, 0.02). Returns (inputs dict, weights dict)."""
    inputs = {}
    for i, key in enumerate(("qkv", "o", "gateup", "down")):
        K = {"qkv": 5120, "o": 8192, "gateup": 5120, "down": 25600}[key]
        inputs[key] = dense_case(1000 * 3 + 100 * sweep + i, M, K, 1, heavy_tail=True, n_outliers=0,
                                 draw_w=False, name=f"qwen3_32b_{key}_M{M}", device=device)
    weights = {}
    if draw_w:
        for j, (name, K, N, _) in enumerate(QWEN3_32B_LINEARS):
            g = _gen(1000 * 3 + 50 + j, device)
            weights[name] = normal_bf16(g, (N, K), 0.02)
    return inputs, weights


@dataclass
class MoECase:
    """Grouped linear: X_perm [sum M_e, K] sorted by expert, offsets int32 [E+1], W [E, N, K], s [E, K].
    routing: the top-k routing; X_tok: the gate/up input in token order [T, K] (X = X_tok[routing.token]),
    None for the down projection, whose input is drawn directly in expert-sorted order."""
    name: str
    X: torch.Tensor
    W: torch.Tensor | None
    s: torch.Tensor
    offsets: torch.Tensor
    had_block: int
    routing: "Routing | None" = None
    X_tok: torch.Tensor | None = None


@dataclass
class Routing:
    """Top-k routing of T tokens over E experts, rows sorted by (expert, token)."""
    token: torch.Tensor     # int64 [T * topk]: the token of each expert-sorted row
    offsets: torch.Tensor   # int32 [E + 1]: rows of expert e are offsets[e] .. offsets[e+1]
    pos: torch.Tensor       # int32 [T, topk]: the sorted row of token t's j-th choice
    weights: torch.Tensor   # fp32 [T, topk]: router weights, softmax over the chosen perturbed scores


def moe_routing_full(g: torch.Generator, T: int, E: int, topk: int, zipf: float = 1.1) -> Routing:
    """Zipf(zipf) expert popularity over ranks, mapped to experts by a seeded permutation; each token
    picks topk distinct experts by Gumbel-top-k on log p. The router weights are the softmax of the
    chosen experts' perturbed scores (no further random draws)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p_rank = ranks ** (-zipf)
    p_rank /= p_rank.sum()
    perm = torch.randperm(E, generator=g)
    logp = torch.empty(E, dtype=torch.float64)
    logp[perm] = torch.log(p_rank)
    u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_min(1e-300)
    gumbel = -torch.log(-torch.log(u))
    top = torch.topk(logp[None, :] + gumbel, topk, dim=1)
    choice = top.indices  # [T, topk]
    expert = choice.reshape(-1)
    token = torch.arange(T).repeat_interleave(topk)
    order = torch.argsort(expert * T + token)  # stable by (expert, token)
    counts = torch.bincount(expert, minlength=E)
    offsets = torch.zeros(E + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    inv = torch.empty_like(order)
    inv[order] = torch.arange(order.numel())
    pos = inv.reshape(T, topk).to(torch.int32)
    weights = torch.softmax(top.values, dim=1).to(torch.float32)
    return Routing(token[order], offsets, pos, weights)


def moe_routing(g: torch.Generator, T: int, E: int, topk: int, zipf: float = 1.1):
    """Zipf(zipf) expert popularity over ranks, mapped to experts by a seeded permutation; each token
    picks topk distinct experts by Gumbel-top-k on log p. Returns (token index per row, offsets)."""
    r = moe_routing_full(g, T, E, topk, zipf)
    return r.token, r.offsets


MOE_30B_A3B = dict(E=128, topk=8, hidden=2048, inter=768)
MOE_T = (64, 1024, 8192)


def moe_30b_a3b(T: int, proj: str = "gate_up", draw_w: bool = True, E: int | None = None) -> MoECase:
    """MoE 30B-A3B-shaped grouped GEMM: 128 experts, top-8 of T tokens, Zipf(1.1) popularity.
    gate_up: X_perm [8T, 2048] (gathered token rows) -> [8T, 1536]; down: a fresh [8T, 768] -> [8T, 2048].
    Per-expert s; 0.5% outlier channels x30; W ~ N(0, 0.02)."""
    cfg = MOE_30B_A3B
    E = E or cfg["E"]
    K, N = (cfg["hidden"], 2 * cfg["inter"]) if proj == "gate_up" else (cfg["inter"], cfg["hidden"])
    idx = MOE_T.index(T) if T in MOE_T else 9
    g = _gen(1000 * 4 + 10 * idx + (0 if proj == "gate_up" else 1))
    s = torch.stack([log_uniform_scale(g, K) for _ in range(E)])
    out = outlier_channels(g, K, round(0.005 * K))
    routing = moe_routing_full(g, T, E, cfg["topk"])
    token, offsets = routing.token, routing.offsets
    sigma = torch.ones(K, dtype=torch.float32)
    sigma[out] *= 30.0
    X_tok = None
    if proj == "gate_up":
        X_tok = (torch.randn(T, K, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)
        X = X_tok[token]
    else:
        X = (torch.randn(token.numel(), K, generator=g, dtype=torch.float32) * sigma).to(torch.bfloat16)
    W = normal_bf16(g, (E, N, K), 0.02) if draw_w else None
    return MoECase(f"moe_30b_a3b_{proj}_T{T}", X, W, s, offsets, 32, routing, X_tok)


PREFILL_M = (4096, 16384)
PREFILL_K = (8192, 16384)
PREFILL_N = (8192, 28672)


def large_prefill(M: int, K: int, N: int, draw_w: bool = True, device: str = "cpu") -> DenseCase:
    """Large prefill dense sweep: X ~ N(0,1) with 0.5% outlier channels x50, W ~ N(0, 0.015)."""
    idx = PREFILL_M.index(M) * 4 + PREFILL_K.index(K) * 2 + PREFILL_N.index(N)
    return dense_case(1000 * 5 + idx, M, K, N, w_std=0.015, n_outliers=round(0.005 * K), outlier_factor=50.0,
                      had_block=32, name=f"prefill_M{M}_K{K}_N{N}", draw_w=draw_w, device=device)
