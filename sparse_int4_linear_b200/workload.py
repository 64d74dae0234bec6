"""Seeded synthetic inputs for the compressed linear layer.

This module only draws random numbers; it holds none of the layer's
arithmetic (no quantization, pruning, packing or matmul).  Both the CPU
oracle's tests and the CUDA path's tests and benchmark take their inputs from
here, so the two sides always see the same bits.

Recipe (shapes of the LLaMA-2-7B / 70B linear layers the thesis evaluates in
its SLiM layer-wise speedup table and figure; synthetic values, because no
trained weights are used):

* one torch CPU generator per layer, ``manual_seed(seed)``; draws in this
  order: W fp32 [N][K] ~ N(0, sigma_w); L [K][r] ~ N(0, 0.01);
  R [r][N] ~ N(0, 0.01); X fp32 [M][K] ~ N(0, 1); outlier channels
  ``randperm(K)[:n_out]`` whose X columns are multiplied by ``out_factor``;
* everything is then rounded to bf16 (round-to-nearest-even) and returned as
  uint16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class LayerSpec:
    name: str
    K: int
    N: int
    r: int
    seed: int
    sigma_w: float = 0.02
    n_out: int = 0
    out_factor: float = 20.0


@dataclass
class LayerInputs:
    spec: LayerSpec
    W: np.ndarray  # uint16 bf16 bits [N][K]
    L: np.ndarray  # uint16 bf16 bits [K][r]
    R: np.ndarray  # uint16 bf16 bits [r][N]
    X: np.ndarray  # uint16 bf16 bits [M][K]


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def make_layer(spec: LayerSpec, M: int) -> LayerInputs:
    g = torch.Generator().manual_seed(int(spec.seed))
    W = torch.randn(spec.N, spec.K, generator=g, dtype=torch.float32) * spec.sigma_w
    L = torch.randn(spec.K, spec.r, generator=g, dtype=torch.float32) * 0.01
    R = torch.randn(spec.r, spec.N, generator=g, dtype=torch.float32) * 0.01
    X = torch.randn(M, spec.K, generator=g, dtype=torch.float32)
    if spec.n_out > 0:
        idx = torch.randperm(spec.K, generator=g)[: spec.n_out]
        X[:, idx] *= spec.out_factor
    return LayerInputs(spec, _bf16_bits(W), _bf16_bits(L), _bf16_bits(R), _bf16_bits(X))


def make_x(K: int, M: int, seed: int, n_out: int = 0, out_factor: float = 20.0) -> np.ndarray:
    """A stand-alone activation batch (same distribution as make_layer's X)."""
    g = torch.Generator().manual_seed(int(seed))
    X = torch.randn(M, K, generator=g, dtype=torch.float32)
    if n_out > 0:
        idx = torch.randperm(K, generator=g)[:n_out]
        X[:, idx] *= out_factor
    return _bf16_bits(X)


def n_outliers(K: int) -> int:
    return int(round(0.01 * K))


# Layer index within a LLaMA decoder block (used in the per-layer seeds).
BLOCK_INDEX = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6}


def _l7(name: str, K: int, N: int, cfg: int) -> LayerSpec:
    return LayerSpec(f"7b.{name}", K, N, 128, 1000 * cfg + BLOCK_INDEX[name], 0.02, n_outliers(K), 20.0)


def _l70(name: str, K: int, N: int) -> LayerSpec:
    return LayerSpec(f"70b.{name}", K, N, 256, 5000 + BLOCK_INDEX[name], 0.015, n_outliers(K), 30.0)


# The five workloads: (layers, token counts M).
CONFIGS = {
    1: ([LayerSpec("tiny", 256, 256, 16, 0, 0.02, 2, 20.0)], [16]),
    2: ([_l7("q", 4096, 4096, 2)], [1, 4, 16]),
    3: ([_l7("up", 4096, 11008, 3), _l7("down", 11008, 4096, 3)], [2048]),
    4: ([_l7("q", 4096, 4096, 4), _l7("k", 4096, 4096, 4), _l7("v", 4096, 4096, 4),
         _l7("o", 4096, 4096, 4), _l7("gate", 4096, 11008, 4), _l7("up", 4096, 11008, 4),
         _l7("down", 11008, 4096, 4)], [1, 16, 256, 1024, 4096]),
    5: ([_l70("q", 8192, 8192), _l70("k", 8192, 1024), _l70("v", 8192, 1024),
         _l70("gate", 8192, 28672), _l70("up", 8192, 28672), _l70("down", 28672, 8192)],
        [1, 16, 512, 4096]),
}
