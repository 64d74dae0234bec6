"""slim_linear_noalloc: the forward for callers that cannot allocate device
memory (an engine plugin whose device memory is planned up front, code where
cudaMalloc is not allowed or would synchronize the device).  Its scratch for
the adapter's X L lives in a fixed array inside the library rather than in a
caller-provided workspace.

It must give what slim_linear gives, and what the fp64 oracle gives.  This
file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
Acceptance as in every parity test: relative Frobenius error <= 5e-3 and
max-abs error <= 2e-2 * max|Y_ref|.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, oracle_reference, sample_rows, to_dev
from sparse_int4_linear_b200.workload import LayerSpec, make_layer

pytestmark = pytest.mark.gpu


def _close(Y, Y_ref, what):
    rel, mab = oracle.errors(Y, Y_ref)
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, f"{what}: rel={rel:.3e} maxabs={mab:.3e}"


def test_noalloc_matches_workspace_entry_point_twice(lib):
    li = make_layer(LayerSpec("noalloc", 4096, 1024, 128, 77, 0.02, 41, 20.0), 16)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = to_dev(li.X)
    for M in (16, 5):                        # two calls in a row, different sizes
        Y_ws = from_dev_bf16(lib.linear(layer, X[:M]))
        Y_na = from_dev_bf16(lib.linear_noalloc(layer, X[:M]))
        torch.cuda.synchronize()
        _close(Y_na, Y_ws, f"noalloc vs slim_linear, M={M}")
    lib.sync_status(layer)


@pytest.mark.parametrize("M", [1, 16, 300, 496])
def test_noalloc_matches_oracle(lib, M):
    """Seeded data at r = 256: the single-launch kernel (M <= 16) and the
    token-tiled kernels up to the largest M the array holds."""
    li = make_layer(LayerSpec("noalloc.r256", 2048, 1024, 256, 5000 + M, 0.015, 20, 30.0), M)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    Y = lib.linear_noalloc(layer, to_dev(li.X))
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _close(from_dev_bf16(Y), oracle_reference(li, li.X), f"noalloc M={M}")


def test_noalloc_across_regimes(lib):
    """The shared array after a token-tiled call (M > 16) serves a
    single-launch call that splits K into several panels and every row tile
    across several warps (its arrival words and segment partials lie where
    the X L of the token-tiled call was)."""
    K, N, r = 32768, 64, 64
    li = make_layer(LayerSpec("noalloc.regimes", K, N, r, 5151, 0.02, K // 100, 20.0), 40)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = to_dev(li.X)
    rows = sample_rows(N, 96, 3)
    assert layer.launches(8) == 1
    outs = [(M, lib.linear_noalloc(layer, X[:M]).clone()) for M in (40, 8, 40, 8)]
    torch.cuda.synchronize()
    lib.sync_status(layer)
    for M, Y in outs:
        _close(from_dev_bf16(Y)[:, rows], oracle_reference(li, li.X[:M], rows), f"noalloc M={M}")


def test_noalloc_rejects_sizes_beyond_its_array(lib):
    li = make_layer(LayerSpec("noalloc", 256, 64, 256, 78, 0.02, 3, 20.0), 512)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    # r = 256: a 256-byte control block + 512 bytes per token of X L in
    # whole 16-token tiles; 256 KB holds 496 tokens, not 512.
    X = to_dev(li.X)
    with pytest.raises(lib.SlimError) as ei:
        lib.linear_noalloc(layer, X)
    assert ei.value.name == "SLIM_ERR_WORKSPACE"
    Y = lib.linear_noalloc(layer, X[:496])
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _close(from_dev_bf16(Y), oracle_reference(li, li.X[:496]), "noalloc M=496")
