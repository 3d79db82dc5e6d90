"""Seeded synthetic inputs for the phase-specialised quantized linear layers.

This module only draws random numbers and lays out shapes.  It holds none of
the quantization arithmetic, so both the CPU oracle (test infrastructure) and
the CUDA path can consume its tensors without sharing any method code.

Workloads follow the layer shapes of the Qwen3 family named on the Mix-Quant
page (gist.science, "Mix-Quant", section 4 "experimental results") and the
"large linear layers" of the MARLIN page (abeam.tech, "experiments and
results").  Activations carry a few large-magnitude channels, the outlier
structure that the KLLM dialogue (aibr.jp, Orizuru discussion) gives as the
reason low-bit activation quantization is hard.

Recipe (all draws on a CPU ``torch.Generator`` in float32, cast once to
bfloat16 with round-to-nearest-even):
  * activations X[M, K] ~ N(0, 1); ``n_outliers`` channels picked by
    ``randperm(K)`` under ``seed + 2`` are multiplied by ``outlier_gain``;
  * weights W[N, K] ~ N(0, 1) * 0.02 under ``seed + 1``.
"""
from __future__ import annotations

import dataclasses

import torch

# Qwen3-8B: hidden 4096, 32 q / 8 kv heads of dim 128, intermediate 12288.
QWEN3_8B_LINEARS = (
    ("qkv_proj", 4096, 6144),
    ("o_proj", 4096, 4096),
    ("gate_up_proj", 4096, 24576),
    ("down_proj", 12288, 4096),
)
# Qwen3-32B: hidden 5120, 64 q / 8 kv heads of dim 128, intermediate 25600.
QWEN3_32B_LINEARS = (
    ("qkv_proj", 5120, 10240),
    ("o_proj", 8192, 5120),
    ("gate_up_proj", 5120, 51200),
    ("down_proj", 25600, 5120),
)
DECODE_BATCHES = (1, 4, 8, 16, 32)
CROSSOVER_BATCHES = (1, 8, 32, 128, 512, 2048, 8192, 32768)


def n_outlier_channels(K: int) -> int:
    """0.1 % of the channels, at least one (4, 12, 5, 8, 26 for the Qwen3 K's)."""
    return max(1, int(round(0.001 * K)))


def activations(M: int, K: int, seed: int, n_outliers: int | None = None,
                outlier_gain: float = 20.0) -> torch.Tensor:
    """BF16 [M, K] ~ N(0,1) with ``n_outliers`` channels scaled by ``outlier_gain``."""
    if n_outliers is None:
        n_outliers = n_outlier_channels(K)
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    gc = torch.Generator(device="cpu").manual_seed(seed + 2)
    ch = torch.randperm(K, generator=gc)[:n_outliers]
    x[:, ch] *= outlier_gain
    return x.to(torch.bfloat16)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """BF16 [N, K] ~ N(0, std^2)."""
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    return (torch.randn(N, K, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def activations_cuda(M: int, K: int, seed: int, device="cuda", n_outliers=None,
                     outlier_gain: float = 20.0) -> torch.Tensor:
    """Same distribution as :func:`activations`, drawn on the GPU (for large bench
    inputs, where a CPU draw would dominate set-up time).  Values differ from the
    CPU draw; parity tests use the CPU draw."""
    if n_outliers is None:
        n_outliers = n_outlier_channels(K)
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32, device=device)
    gc = torch.Generator(device="cpu").manual_seed(seed + 2)
    ch = torch.randperm(K, generator=gc)[:n_outliers].to(device)
    x[:, ch] *= outlier_gain
    return x.to(torch.bfloat16)


def weights_cuda(N: int, K: int, seed: int, device="cuda", std: float = 0.02) -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(seed + 1)
    return (torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * std).to(torch.bfloat16)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    seed: int


def tiny_case() -> tuple[torch.Tensor, torch.Tensor]:
    """The tiny correctness case: X [128, 512] with 4 outlier channels, W [512, 512], seed 0."""
    return activations(128, 512, seed=0, n_outliers=4), weights(512, 512, seed=0)


def prefill_workloads(M: int, linears, seed_base: int) -> list[Workload]:
    return [Workload(name, M, K, N, seed_base + 10 * i) for i, (name, K, N) in enumerate(linears)]
