"""Seeded synthetic inputs for BitLinear workloads.

This module only draws random numbers and names shapes; it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from
it.  Everything is generated on the host with a torch CPU generator so the
same seed gives the same bytes on every machine.

Recipe (BitNet-b1.58-style layers):
  * latent weights  W ~ N(0, 0.02), binary32                     (per matrix seed)
  * activations     x ~ N(0, 1); with ``outliers`` an independent mask
                    (uniform < 0.01, seed + 1) scales 1% of entries by 20;
                    then cast to the requested dtype
  * RMSNorm gain    all ones
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

W_SIGMA = 0.02
OUTLIER_FRAC = 0.01
OUTLIER_MULT = 20.0

HIDDEN = 2560
FFN = 6912
N_LAYERS = 30


def latent_weights(N: int, K: int, seed: int, sigma: float = W_SIGMA) -> torch.Tensor:
    """Latent full-precision weights W [N, K] ~ N(0, sigma), float32, CPU."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn((N, K), generator=g, dtype=torch.float32) * sigma


def activations(M: int, K: int, seed: int, outliers: bool = True,
                dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Activations x [M, K] ~ N(0, 1) with optional 1% x20 outliers, CPU."""
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn((M, K), generator=g, dtype=torch.float32)
    if outliers:
        g2 = torch.Generator().manual_seed(int(seed) + 1)
        mask = torch.rand((M, K), generator=g2) < OUTLIER_FRAC
        x = torch.where(mask, x * OUTLIER_MULT, x)
    return x.to(dtype)


def unit_gain(K: int) -> torch.Tensor:
    return torch.ones(K, dtype=torch.float32)


@dataclass(frozen=True)
class Matrix:
    name: str
    K: int       # in-features
    N: int       # out-features
    seed: int


def layer_matrices(layer: int, hidden: int = HIDDEN, ffn: int = FFN):
    """The seven BitLinear matrices of one transformer block, in call order:
    Q, K, V, O (hidden -> hidden), up and gate (hidden -> ffn), down (ffn -> hidden).
    Seeds are 1000 * layer + matrix index."""
    shapes = [("q", hidden, hidden), ("k", hidden, hidden), ("v", hidden, hidden),
              ("o", hidden, hidden), ("up", hidden, ffn), ("gate", hidden, ffn),
              ("down", ffn, hidden)]
    return [Matrix(f"L{layer}.{n}", K, N, 1000 * layer + i) for i, (n, K, N) in enumerate(shapes)]


def stack_matrices(n_layers: int = N_LAYERS):
    out = []
    for layer in range(n_layers):
        out.extend(layer_matrices(layer))
    return out


# Decode GEMV shapes (K, N) of one block: attention projections, FFN up, FFN down.
DECODE_SHAPES = [(HIDDEN, HIDDEN), (HIDDEN, FFN), (FFN, HIDDEN)]
# Prefill/batched sweep at K = 2560, N = 6912.
SWEEP_M = [1, 4, 16, 64, 256, 1024, 4096]
# 70B-class FFN shapes (K, N) and token counts.
LARGE_SHAPES = [(8192, 28672), (28672, 8192)]
LARGE_M = [1, 8, 512]
