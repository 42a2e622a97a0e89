"""Seeded synthetic inputs shaped like the pages' weights and KV caches.

This module holds input recipes only -- distributions, shapes and seeds -- and
none of the quantizer's arithmetic.  It is the one module that both the CUDA
path's tests/benchmark and the CPU oracle's callers share.  Every generator
takes an explicit seed and device and returns torch tensors in the stated
16-bit dtype; the same bytes are then handed to both sides.

Recipes (one per workload):
  * ``gaussian_matrix``      fp16/bf16 i.i.d. N(0, std^2)                     (256 x 512 fp16 weight)
  * ``student_t_outliers``   Student-t nu=4 scaled to std 0.02, with exactly
                             round(0.001 * N) distinct random positions x20     (4096 x 4096 bf16 weight)
  * ``llama_linear``         N(0, 0.02^2) times a per-output-row scale
                             exp(U[ln 0.5, ln 2])                              (Llama-7B decoder linears)
  * ``kv_with_channels``     N(0,1) with 4 fixed channels per head x10          (KV cache, head_dim 128)
  * ``normal``               plain N(0,1)                                      (keys / queries)
"""
from __future__ import annotations

import math

import torch

LLAMA7B_LINEARS = (
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_matrix(rows: int, cols: int, std: float, seed: int, dtype=torch.float16, device="cpu"):
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    return x.to(dtype)


def student_t_outliers(rows: int, cols: int, seed: int, std: float = 0.02, nu: int = 4,
                       outlier_frac: float = 0.001, outlier_mult: float = 20.0,
                       dtype=torch.bfloat16, device="cpu"):
    """t_nu = Z / sqrt(chi2_nu / nu) with chi2_nu a sum of nu squared normals;
    var(t_nu) = nu / (nu - 2), so the draw is scaled by std / sqrt(nu/(nu-2))."""
    g = _gen(seed, device)
    n = rows * cols
    z = torch.randn(n, generator=g, device=device, dtype=torch.float32)
    chi = torch.zeros(n, device=device, dtype=torch.float32)
    for _ in range(nu):
        e = torch.randn(n, generator=g, device=device, dtype=torch.float32)
        chi += e * e
    t = z / torch.sqrt(chi / nu)
    t *= std / math.sqrt(nu / (nu - 2))
    k = int(round(outlier_frac * n))
    pos = torch.randperm(n, generator=g, device=device)[:k]
    t[pos] *= outlier_mult
    return t.view(rows, cols).to(dtype)


def llama_linear(rows: int, cols: int, seed: int, std: float = 0.02, dtype=torch.bfloat16, device="cpu"):
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    u = torch.rand(rows, 1, generator=g, device=device, dtype=torch.float32)
    scale = torch.exp(math.log(0.5) + u * (math.log(2.0) - math.log(0.5)))
    return (w * scale).to(dtype)


def kv_with_channels(batch: int, heads: int, seq: int, head_dim: int, seed: int, n_channels: int = 4,
                     mult: float = 10.0, dtype=torch.bfloat16, device="cpu"):
    """[batch][heads][seq][head_dim] N(0,1); per head, n_channels channels
    (drawn once from the seed, the same for every batch and token) x mult."""
    g = _gen(seed, device)
    x = torch.randn(batch, heads, seq, head_dim, generator=g, device=device, dtype=torch.float32)
    gc = _gen(seed + 7919, "cpu")
    scale = torch.ones(heads, head_dim, dtype=torch.float32)
    for h in range(heads):
        ch = torch.randperm(head_dim, generator=gc)[:n_channels]
        scale[h, ch] = mult
    x *= scale.to(device).view(1, heads, 1, head_dim)
    return x.to(dtype)


def normal(shape, seed: int, dtype=torch.bfloat16, device="cpu"):
    g = _gen(seed, device)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def as_u16(t: torch.Tensor):
    """16-bit tensor -> numpy uint16 bit patterns on the host (for the oracle)."""
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
