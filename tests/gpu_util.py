"""Helpers shared by the GPU parity tests (oracle side computed on the CPU)."""
import numpy as np
import torch

import oracle


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit array -> bf16 CUDA tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> float64 numpy (exact)."""
    return t.float().cpu().numpy().astype(np.float64)


def oracle_rows(W_bits, rows):
    """Oracle pack of selected rows only (quantization and pruning are row-local)."""
    return oracle.pack_layer(np.ascontiguousarray(W_bits[rows]))


def oracle_reference(li, X_bits, rows=None):
    """fp64 Y_ref [M][len(rows)] for the selected output rows (all rows if None)."""
    W = li.W if rows is None else li.W[rows]
    vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(W))
    if li.spec.r:
        R = li.R if rows is None else li.R[:, rows]
        return oracle.forward(vals, meta, sc, li.L, np.ascontiguousarray(R), X_bits)
    return oracle.forward(vals, meta, sc, None, None, X_bits)


def sample_rows(N, n, seed=0):
    rng = np.random.default_rng(seed)
    if N <= n:
        return np.arange(N)
    rows = np.sort(rng.choice(N, size=n, replace=False))
    # always include the first and last row (tile edges)
    return np.unique(np.concatenate([[0, N - 1], rows]))
