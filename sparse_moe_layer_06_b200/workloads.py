"""Seeded synthetic workloads for the sparse MoE FFN layer.

This module only names the layer shapes and draws the random inputs; it holds
none of the layer's arithmetic, so both the CUDA path's tests/benchmark and the
CPU oracle can take their inputs from it.

Shapes and constants (page "Hy4 preview config.json 终极深度解读", section
"MoE 路由专家256 选 8" and the spec table: hidden_size 6144, n_routed_experts
256, num_experts_per_tok 8, n_shared_experts 1, moe_intermediate_size 2048,
routed_scaling_factor 2.827, swiglu_limit 10.0, initializer_range 0.006,
bfloat16; page "腾讯混元Hy3正式版深度解析", SparseMoERouter sketch: hidden 7168,
32 experts, top-2).

Recipe: every tensor is drawn fp32 N(0, std) from its own ``torch.Generator``
seeded ``seed + j`` (x: j=0, gate weight: j=1, expert weights: j=2, shared
expert: j=3) on the requested device, then cast to the layer dtype.  Expert
weights are drawn one expert at a time (bounded temporary memory).  The skewed
workload adds a fixed per-expert logit bias 0.5*ln(p_e), p_e proportional to
(e+1)^-1.2 (a Zipf(1.2) share profile), so a few experts take >10% of tokens.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # routed experts
    top_k: int        # experts per token
    I: int            # expert intermediate size
    num_shared: int   # 0 or 1 shared experts (width I)
    dtype: torch.dtype
    x_std: float
    w_std: float
    routed_scale: float
    clip_limit: float  # <= 0: no clamp
    skew_bias: bool = False
    description: str = ""

    def with_tokens(self, T: int) -> "MoEConfig":
        return replace(self, T=T)


CONFIGS: dict[str, MoEConfig] = {
    "tiny": MoEConfig(
        "tiny", T=64, H=256, E=16, top_k=2, I=128, num_shared=1, dtype=torch.float32,
        x_std=1.0, w_std=0.02, routed_scale=2.827, clip_limit=10.0,
        description="tiny MoE layer: T=64, H=256, E=16 top-2 + 1 shared, I=128, fp32"),
    "hy3": MoEConfig(
        "hy3", T=2048, H=7168, E=32, top_k=2, I=2048, num_shared=0, dtype=torch.bfloat16,
        x_std=1.0, w_std=0.006, routed_scale=1.0, clip_limit=0.0,
        description="Hy3-shape MoE layer: T=2048, H=7168, E=32 top-2, I=2048, no shared, bf16"),
    "hy4_prefill": MoEConfig(
        "hy4_prefill", T=4096, H=6144, E=256, top_k=8, I=2048, num_shared=1,
        dtype=torch.bfloat16, x_std=1.0, w_std=0.006, routed_scale=2.827, clip_limit=10.0,
        description="Hy4-shape prefill MoE layer: T=4096, H=6144, E=256 top-8 + 1 shared, "
                    "I=2048, bf16"),
    "hy4_decode": MoEConfig(
        "hy4_decode", T=64, H=6144, E=256, top_k=8, I=2048, num_shared=1,
        dtype=torch.bfloat16, x_std=1.0, w_std=0.006, routed_scale=2.827, clip_limit=10.0,
        description="Hy4-shape decode MoE layer: T=64, H=6144, E=256 top-8 + 1 shared, "
                    "I=2048, bf16"),
    "hy4_skew": MoEConfig(
        "hy4_skew", T=16384, H=6144, E=256, top_k=8, I=2048, num_shared=1,
        dtype=torch.bfloat16, x_std=1.0, w_std=0.006, routed_scale=2.827, clip_limit=10.0,
        skew_bias=True,
        description="Hy4-shape skewed routing: T=16384, E=256 top-8 + 1 shared, "
                    "Zipf(1.2) logit bias"),
}


def skew_logit_bias(E: int) -> torch.Tensor:
    """Per-expert logit bias 0.5*ln((e+1)^-1.2), fp32 [E] (input recipe)."""
    return torch.tensor([0.5 * (-1.2) * math.log(e + 1.0) for e in range(E)],
                        dtype=torch.float32)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, dtype, device, gen) -> torch.Tensor:
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
            .mul_(std).to(dtype))


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu") -> dict:
    """Draw x, gate_w, expert_w [E,3,I,H], shared_w [3,I,H] (or None), logit_bias."""
    device = torch.device(device)
    x = _normal((cfg.T, cfg.H), cfg.x_std, cfg.dtype, device, _gen(device, seed + 0))
    gate_w = _normal((cfg.E, cfg.H), cfg.w_std, cfg.dtype, device, _gen(device, seed + 1))
    g2 = _gen(device, seed + 2)
    expert_w = torch.empty((cfg.E, 3, cfg.I, cfg.H), dtype=cfg.dtype, device=device)
    for e in range(cfg.E):
        expert_w[e] = _normal((3, cfg.I, cfg.H), cfg.w_std, cfg.dtype, device, g2)
    shared_w = None
    if cfg.num_shared:
        shared_w = _normal((3, cfg.I, cfg.H), cfg.w_std, cfg.dtype, device,
                           _gen(device, seed + 3))
    bias = skew_logit_bias(cfg.E).to(device) if cfg.skew_bias else None
    return dict(x=x, gate_w=gate_w, expert_w=expert_w, shared_w=shared_w, logit_bias=bias)


def make_router_inputs(cfg: MoEConfig, seed: int = 0, device="cpu") -> dict:
    """Only x, gate_w and logit_bias of make_inputs (same draws), without the
    expert weights."""
    device = torch.device(device)
    x = _normal((cfg.T, cfg.H), cfg.x_std, cfg.dtype, device, _gen(device, seed + 0))
    gate_w = _normal((cfg.E, cfg.H), cfg.w_std, cfg.dtype, device, _gen(device, seed + 1))
    bias = skew_logit_bias(cfg.E).to(device) if cfg.skew_bias else None
    return dict(x=x, gate_w=gate_w, logit_bias=bias)


def make_x(cfg: MoEConfig, seed: int = 0, device="cpu") -> torch.Tensor:
    """Only the token activations of make_inputs (same draw)."""
    device = torch.device(device)
    return _normal((cfg.T, cfg.H), cfg.x_std, cfg.dtype, device, _gen(device, seed + 0))


def sample_tokens(T: int, n: int, seed: int = 0):
    """A seeded, sorted subset of n token indices out of T (all if n >= T)."""
    if n >= T:
        return list(range(T))
    g = _gen("cpu", seed + 1000)
    return sorted(torch.randperm(T, generator=g)[:n].tolist())
