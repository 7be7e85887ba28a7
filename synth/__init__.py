"""Seeded synthetic inputs for the NVFP4 linear layer workloads.

This module only draws random numbers; it holds none of the quantization or GEMM arithmetic.
Both the CPU oracle (through the tests) and the CUDA path consume what it returns, so the two
sides see the same bytes.

Recipe (all values drawn on the host with ``torch.Generator('cpu').manual_seed(seed)`` as
fp32 ``randn``, scaled by the standard deviation, then rounded to bf16 round-to-nearest-even):

- activations X [T][d] ~ N(0, 1); optionally a fraction of the d channels (the first
  ``n_outlier`` entries of ``randperm(d)`` under ``outlier_seed``) multiplied by 50 before the
  bf16 rounding -- the outlier channels the pages give as the reason for the Hadamard rotation;
- weights W [n][d] ~ N(0, 0.02);
- output gradients dY [T][n] ~ N(0, 1e-4).

The second parameter of N(., .) is the standard deviation.
"""
from __future__ import annotations

import torch

# Shapes of the 12B-hybrid-sized MLP up-projection the workloads are quoted on.
TOKENS = 8192
D_IN = 5120
D_OUT = 20480


def normal_bf16(rows: int, cols: int, std: float, seed: int) -> torch.Tensor:
    """[rows][cols] bf16 (CPU), N(0, std) drawn under ``seed``."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn((rows, cols), generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def activations(tokens: int, d: int, seed: int = 0, outlier_frac: float = 0.0,
                outlier_scale: float = 50.0, outlier_seed: int = 10) -> torch.Tensor:
    """X [tokens][d] bf16 ~ N(0, 1) with ``round(outlier_frac * d)`` channels scaled by 50."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn((tokens, d), generator=g, dtype=torch.float32)
    n_out = int(round(outlier_frac * d))
    if n_out > 0:
        go = torch.Generator(device="cpu").manual_seed(int(outlier_seed))
        cols = torch.randperm(d, generator=go)[:n_out]
        x[:, cols] *= outlier_scale
    return x.to(torch.bfloat16)


def weights(n: int, d: int, seed: int = 1, std: float = 0.02) -> torch.Tensor:
    return normal_bf16(n, d, std, seed)


def grad_output(tokens: int, n: int, seed: int = 2, std: float = 1e-4) -> torch.Tensor:
    return normal_bf16(tokens, n, std, seed)


def bf16_bits(t: torch.Tensor):
    """The raw uint16 bit patterns of a CPU bf16 tensor as a numpy array (no copy of values)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def sample_indices(m: int, n: int, count: int, seed: int):
    """``count`` seeded random (row, col) output positions in an m x n result."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    ii = torch.randint(0, m, (count,), generator=g, dtype=torch.int64)
    jj = torch.randint(0, n, (count,), generator=g, dtype=torch.int64)
    return ii.numpy(), jj.numpy()
