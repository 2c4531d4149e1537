"""Seeded synthetic inputs for the quantization workloads.

This module only draws random tensors; it holds none of the quantization
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.
Every generator is deterministic in its ``seed`` and runs on the CPU with a
private ``torch.Generator`` (or, for the Student-t draw, a forked global RNG),
so the global RNG state of the caller is left untouched.

Shapes default to the five benchmark workloads; smaller shapes keep the same
value distribution for fast parity tests.

* ``glossary_example``  -- the Ultralytics glossary "FP4" worked example:
  ``torch.manual_seed(0); randn(4096)`` with every 512th value times 20.
* ``small_matrix``      -- 256x256 BF16, N(0,1), every 512th flat value x20.
* ``activation``        -- tokens x hidden BF16, N(0,1), a few seeded outlier
  columns scaled x50.
* ``weight``            -- FP32 master weight, N(0, 0.02), 0.01% of entries x30.
* ``gradient``          -- BF16 Student-t(nu=3) * 1e-3 output gradient.
* ``if4_blocks``        -- BF16 rows of 16-value blocks, half U(-1,1) and half
  Laplace(0,1), one x10 outlier per block.
"""
from __future__ import annotations

import torch

__all__ = ["glossary_example", "small_matrix", "activation", "weight", "gradient",
           "if4_blocks", "WORKLOADS"]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def glossary_example() -> torch.Tensor:
    """FP32 [4096]: seed 0, N(0,1), x[::512] *= 20 (the glossary's snippet input)."""
    x = torch.randn(4096, generator=_gen(0), dtype=torch.float32)
    x[::512] *= 20
    return x


def small_matrix(seed: int = 0, rows: int = 256, cols: int = 256) -> torch.Tensor:
    """BF16 [rows, cols]: N(0,1) with every 512th flat element x20.

    At 256x256 with seed 0 its first 4096 values equal the glossary example."""
    x = torch.randn(rows, cols, generator=_gen(seed), dtype=torch.float32)
    x.view(-1)[::512] *= 20
    return x.to(torch.bfloat16)


def activation(seed: int = 0, rows: int = 8192, cols: int = 4096, n_outlier_cols: int = 8,
               outlier_scale: float = 50.0) -> torch.Tensor:
    """BF16 activation X [tokens, hidden]: N(0,1), n_outlier_cols seeded columns x50."""
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    idx = torch.randperm(cols, generator=g)[:n_outlier_cols]
    x[:, idx] *= outlier_scale
    return x.to(torch.bfloat16)


def weight(seed: int = 0, rows: int = 14336, cols: int = 4096, std: float = 0.02,
           outlier_fraction: float = 1e-4, outlier_scale: float = 30.0) -> torch.Tensor:
    """FP32 master weight [out, in]: N(0, std^2), round(fraction*N) seeded entries x30."""
    g = _gen(seed)
    w = torch.randn(rows, cols, generator=g, dtype=torch.float32) * std
    n = rows * cols
    k = int(round(outlier_fraction * n))
    if k > 0:
        idx = torch.randperm(n, generator=g)[:k]
        w.view(-1)[idx] *= outlier_scale
    return w


def gradient(seed: int = 0, tokens: int = 8192, cols: int = 5120, nu: float = 3.0,
             scale: float = 1e-3) -> torch.Tensor:
    """BF16 output gradient dY [tokens, cols]: Student-t(nu) * scale."""
    with torch.random.fork_rng(devices=[]):
        torch.manual_seed(seed)
        t = torch.distributions.StudentT(torch.tensor(float(nu))).sample((tokens, cols))
    return (t * scale).to(torch.bfloat16)


def if4_blocks(seed: int = 0, rows: int = 16384, cols: int = 8192,
               outlier_scale: float = 10.0) -> torch.Tensor:
    """BF16 [rows, cols] of 16-value blocks along rows.

    Each block is, by a seeded coin, either U(-1,1) or Laplace(0,1); one seeded
    position per block is multiplied by 10."""
    assert cols % 16 == 0
    g = _gen(seed)
    nb = rows * cols // 16
    is_laplace = torch.rand(nb, generator=g) < 0.5
    u = torch.rand(nb, 16, generator=g, dtype=torch.float32) * 2.0 - 1.0       # U(-1, 1)
    # Laplace(0, 1) = random sign * Exp(1); Exp(1) = -log(1 - U) with U in [0, 1)
    # stays finite (1 - U >= 2^-24)
    e = -torch.log1p(-torch.rand(nb, 16, generator=g, dtype=torch.float32))
    lap = torch.where(torch.rand(nb, 16, generator=g) < 0.5, -e, e)
    x = torch.where(is_laplace[:, None], lap, u)
    pos = torch.randint(0, 16, (nb,), generator=g)
    x[torch.arange(nb), pos] *= outlier_scale
    return x.reshape(rows, cols).to(torch.bfloat16)


# name -> (generator, full-size kwargs) of the benchmark workloads
WORKLOADS = {
    "small": (small_matrix, {}),
    "activation": (activation, {}),
    "weight": (weight, {}),
    "gradient": (gradient, {}),
    "if4": (if4_blocks, {}),
}
