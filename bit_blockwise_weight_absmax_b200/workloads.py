"""Seeded synthetic inputs shared by the tests, the bench and the smoke run.

This module holds no arithmetic of the quantization method: it only draws
random 16-bit tensors with the shapes and distributions of the workloads
(Gaussian weights, a sprinkling of x20 outliers, Gaussian activations).  No
real checkpoint is used: the "Llama-2-7B" and "Llama-70B" names are shape
templates only.
"""
from __future__ import annotations

import torch

# Linear layers of one Llama-2-7B decoder layer, nn.Linear convention [out, in].
LAYER_7B = [
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
]
# Linear layers of one Llama-70B decoder layer (grouped-query k/v).
LAYER_70B = [
    ("q_proj", 8192, 8192), ("k_proj", 1024, 8192), ("v_proj", 1024, 8192),
    ("o_proj", 8192, 8192), ("gate_proj", 28672, 8192), ("up_proj", 28672, 8192),
    ("down_proj", 8192, 28672),
]
N_LAYERS_70B = 80


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian(shape, std: float, dtype: torch.dtype, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from a seeded generator, then one cast to dtype."""
    x = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def tiny_weight(seed: int = 0) -> torch.Tensor:
    """fp16 W[256, 512] ~ N(0, 0.02)."""
    return gaussian((256, 512), 0.02, torch.float16, seed)


def tiny_activation(seed: int = 1) -> torch.Tensor:
    """fp16 x[1, 512] ~ N(0, 1)."""
    return gaussian((1, 512), 1.0, torch.float16, seed)


def outlier_weight(rows: int = 4096, cols: int = 4096, seed: int = 0, frac: float = 0.001,
                   factor: float = 20.0, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """W ~ N(0, 0.02) with round(frac * n) entries (first indices of a seeded
    permutation) multiplied by `factor` in fp32 before the cast."""
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(0.02)
    n = rows * cols
    k = int(round(frac * n))
    idx = torch.randperm(n, generator=g, device=device)[:k]
    w.view(-1)[idx] *= factor
    return w.to(dtype)


def layer_weights(shapes, std: float, seed: int, dtype=torch.bfloat16, device="cpu"):
    """One weight per (name, N, K) entry, seed + index each."""
    return [gaussian((N, K), std, dtype, seed + i, device) for i, (_, N, K) in enumerate(shapes)]


def activation(M: int, K: int, dtype, seed: int, device="cpu") -> torch.Tensor:
    return gaussian((M, K), 1.0, dtype, seed, device)


# Decoder-only model layouts for the memory-footprint checks (shape templates
# only; no weights): hidden size, MLP size, layers, attention heads, KV heads,
# vocabulary, whether the output head shares the embedding matrix.
# A 135M-class small model (the scale of the demo on
# learn.pranaymahendrakar.com, "Loading a model in 4-bit", "The walkthrough":
# 269 MB at fp16) and the Llama-70B-shaped stack of LAYER_70B.
LAYOUT_135M = dict(hidden=576, inter=1536, layers=30, heads=9, kv_heads=3, vocab=49152, tied=True)
LAYOUT_70B = dict(hidden=8192, inter=28672, layers=N_LAYERS_70B, heads=64, kv_heads=8, vocab=32000,
                  tied=False)
