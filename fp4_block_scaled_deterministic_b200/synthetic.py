"""Seeded synthetic inputs for the 4-bit linear-layer workloads.

This module holds no arithmetic of the method (no rotation, no scaling, no
encoding): it only draws bf16 tensors with the shapes and value distributions
of the workloads, so that the CUDA path and the CPU oracle can be fed the same
bytes. It imports nothing else from this package.

Recipe (all draws from one ``torch.Generator`` per tensor, seeded explicitly):
  * ``normal``: fp32 N(0, std^2), outlier channels = the first
    ``max(1, round(frac * cols))`` entries of ``randperm(cols)`` drawn from the
    same generator, multiplied by ``mult``; then rounded to bf16 (RNE).
  * ``heavy_tailed_grad``: fp32 N(0, std^2); a Bernoulli(p) mask from the same
    generator marks entries replaced by ``std * mult * t`` with t Student-t with
    3 degrees of freedom (t = Z / sqrt(chi2_3 / 3), chi2_3 a sum of three squared
    normals); then bf16.
"""
from __future__ import annotations

import torch

# Llama-3.1-8B layer shapes (N out-features, K in-features) and token count.
LLAMA_TOKENS = 8192  # batch 8 x sequence 1024
LLAMA_LAYERS = (("qkv", 6144, 4096), ("o", 4096, 4096), ("gate", 14336, 4096),
                ("up", 14336, 4096), ("down", 4096, 14336))
# GPT-3 175B layer shapes and token count.
GPT3_TOKENS = 4096
GPT3_LAYERS = (("qkv", 36864, 12288), ("o", 12288, 12288), ("fc1", 49152, 12288),
               ("fc2", 12288, 49152))


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(rows: int, cols: int, std: float = 1.0, seed: int = 0, outlier_frac: float = 0.0,
           outlier_mult: float = 1.0, device="cpu", generator: torch.Generator | None = None):
    g = generator if generator is not None else _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if outlier_frac > 0.0 and cols > 0:
        n_out = max(1, int(round(outlier_frac * cols)))
        idx = torch.randperm(cols, generator=g, device=device)[:n_out]
        x[:, idx] *= outlier_mult
    return x.to(torch.bfloat16)


def heavy_tailed_grad(rows: int, cols: int, std: float = 1e-3, seed: int = 1, p: float = 0.005,
                      mult: float = 20.0, device="cpu"):
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(std)
    mask = torch.rand(rows, cols, generator=g, device=device) < p
    z = torch.randn(rows, cols, generator=g, device=device)
    chi2 = torch.zeros(rows, cols, device=device)
    for _ in range(3):
        chi2.add_(torch.randn(rows, cols, generator=g, device=device).square_())
    t = z / torch.sqrt(chi2 / 3.0)
    x = torch.where(mask, t.mul_(std * mult), x)
    return x.to(torch.bfloat16)


def tiny_linear(device="cpu"):
    """X, W 256x256 N(0,1) from seed 0; 1% of X's columns (3) scaled x30."""
    g = _gen(0, device)
    X = normal(256, 256, 1.0, outlier_frac=0.01, outlier_mult=30.0, device=device, generator=g)
    W = normal(256, 256, 1.0, device=device, generator=g)
    return X, W


def llama_layer(name: str, device="cpu", tokens: int = LLAMA_TOKENS, seed: int = 0):
    """(X [M][K], W [N][K], dY [M][N]) for one Llama-3.1-8B projection: X N(0,1) with
    0.1% outlier channels x50, W N(0, 0.02^2), dY N(0, 1e-3^2) with 0.5% heavy-tailed
    entries (Student-t nu=3, x20)."""
    N, K = dict((n, (a, b)) for n, a, b in LLAMA_LAYERS)[name]
    X = normal(tokens, K, 1.0, seed=seed, outlier_frac=0.001, outlier_mult=50.0, device=device)
    W = normal(N, K, 0.02, seed=seed + 100, device=device)
    dY = heavy_tailed_grad(tokens, N, 1e-3, seed=seed + 200, device=device)
    return X, W, dY


def gpt3_layer(name: str, device="cpu", tokens: int = GPT3_TOKENS, seed: int = 0):
    """(X, W, dY) for one GPT-3 175B projection: X N(0,1) with 0.1% outlier channels
    x100, W N(0, 0.02^2), dY as for Llama."""
    N, K = dict((n, (a, b)) for n, a, b in GPT3_LAYERS)[name]
    X = normal(tokens, K, 1.0, seed=seed, outlier_frac=0.001, outlier_mult=100.0, device=device)
    W = normal(N, K, 0.02, seed=seed + 100, device=device)
    dY = heavy_tailed_grad(tokens, N, 1e-3, seed=seed + 200, device=device)
    return X, W, dY


def sweep_shape(p: int, row_len: int):
    """Rows x row_len for a 2^p-element sweep tensor: rows = 32*max(1, round(2^p/(32 L)))."""
    rows = 32 * max(1, int(round((1 << p) / (32 * row_len))))
    return rows, row_len


def sweep_tensor(p: int, row_len: int, seed: int = 0, device="cpu"):
    rows, cols = sweep_shape(p, row_len)
    return normal(rows, cols, 1.0, seed=seed, outlier_frac=0.001, outlier_mult=50.0, device=device)
