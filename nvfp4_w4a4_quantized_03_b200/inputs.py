"""Seeded synthetic inputs shaped like Qwen3-8B prefill projections.

This module only draws random numbers and casts them to bf16; it contains
none of the quantizer's or the GEMM's arithmetic.  The tests feed the same
tensors to the CUDA path and to the CPU oracle, and the benchmark uses them
as its workload.

The pages evaluate on public benchmarks with trained weights ("Mix-Quant：面向
智能体LLM的量化预填充与精确解码", section 复现评估), which are not available
here; these synthetic tensors stand in for the activations and weights of the
linear layers that run during prefill:
  * activations: N(0, 1) in fp32 with a few outlier channels multiplied by a
    constant, then rounded to bf16;
  * long-context activations: Student-t (nu = 4) scaled per channel by a
    LogNormal(0, 1) factor;
  * weights: N(0, 0.02^2).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

HIDDEN = 4096          # Qwen3-8B hidden size
FFN = 12288            # Qwen3-8B intermediate size
Q_HEADS, KV_HEADS, HEAD_DIM = 32, 8, 128


@dataclasses.dataclass(frozen=True)
class Projection:
    name: str
    K: int   # input features (contraction)
    N: int   # output features


# The four linear layers of one Qwen3-8B decoder layer (QKV and gate/up fused).
QWEN3_8B_PROJECTIONS = (
    Projection("qkv", HIDDEN, (Q_HEADS + 2 * KV_HEADS) * HEAD_DIM),   # 4096 -> 6144
    Projection("o", Q_HEADS * HEAD_DIM, HIDDEN),                      # 4096 -> 4096
    Projection("gate_up", HIDDEN, 2 * FFN),                           # 4096 -> 24576
    Projection("down", FFN, HIDDEN),                                  # 12288 -> 4096
)

# Shape sweep: (K, N) pairs and token counts
SWEEP_KN = ((4096, 4096), (4096, 12288), (12288, 4096), (5120, 25600))
SWEEP_M = (512, 2048, 8192, 32768, 131072)


def outlier_count(K: int, fraction: float = 0.01) -> int:
    return int(round(fraction * K))


def activation_bf16(M: int, K: int, seed: int, outlier_channels: int = 0,
                    outlier_scale: float = 50.0, device: str = "cpu") -> torch.Tensor:
    """N(0,1) activations [M, K] with `outlier_channels` columns scaled up."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32, device=device)
    if outlier_channels:
        idx = torch.randperm(K, generator=g, device=device)[:outlier_channels]
        x[:, idx] *= outlier_scale
    return x.to(torch.bfloat16)


def weight_bf16(N: int, K: int, seed: int, std: float = 0.02, device: str = "cpu") -> torch.Tensor:
    """N(0, std^2) weights [N, K] (nn.Linear layout: out_features x in_features)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return (torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * std).to(torch.bfloat16)


def student_t_activation_bf16(M: int, K: int, seed: int, nu: float = 4.0, device: str = "cpu") -> torch.Tensor:
    """Heavy-tailed activations: X[m, k] = s_k * t[m, k], t ~ Student-t(nu),
    s_k ~ LogNormal(0, 1) per channel (input channel k).  On the CPU the
    draws come from numpy's default_rng(seed); on a GPU from a torch generator
    of that device seeded with `seed` (same distribution, t = z / sqrt(g / nu)
    with z ~ N(0, 1) and g ~ chi-square(nu) = 2 Gamma(nu / 2), another stream
    of numbers), for sizes the host would take long to draw."""
    if str(device) != "cpu":
        g = torch.Generator(device=device).manual_seed(seed)
        s = torch.exp(torch.randn(K, generator=g, device=device))
        z = torch.randn(M, K, generator=g, device=device)
        chi2 = 2.0 * torch._standard_gamma(torch.full((M, K), nu / 2.0, device=device), generator=g)
        return (z * torch.rsqrt(chi2 / nu) * s[None, :]).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    s = rng.lognormal(0.0, 1.0, size=K).astype(np.float32)
    t = rng.standard_t(nu, size=(M, K)).astype(np.float32)
    return torch.from_numpy(t * s[None, :]).to(torch.bfloat16)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a CPU bf16 tensor (no copy of values)."""
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)
