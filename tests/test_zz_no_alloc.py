"""slim_linear_noalloc: the forward for callers that cannot allocate device
memory (its adapter scratch lives in a fixed array inside the library rather
than in a caller-provided workspace).

It must give what slim_linear gives.  This file is collected last so that a
run stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, to_dev
from sparse_int4_linear_b200.workload import LayerSpec, make_layer

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice(lib):
    li = make_layer(LayerSpec("noalloc", 4096, 1024, 128, 77, 0.02, 41, 20.0), 16)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = to_dev(li.X)
    for M in (16, 5):                        # two calls in a row, different sizes
        Y_ws = from_dev_bf16(lib.linear(layer, X[:M]))
        Y_na = from_dev_bf16(lib.linear_noalloc(layer, X[:M]))
        torch.cuda.synchronize()
        rel, mab = oracle.errors(Y_na, Y_ws)
        assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, (M, rel, mab)
    lib.sync_status(layer)


def test_noalloc_rejects_sizes_beyond_its_array(lib):
    li = make_layer(LayerSpec("noalloc", 256, 64, 256, 78, 0.02, 0, 1.0), 1)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    # r = 256: a 256-byte control block + 512 bytes per token of X L in
    # whole 16-token tiles; 256 KB holds 496 tokens, not 512.
    X = torch.zeros(512, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.SlimError) as ei:
        lib.linear_noalloc(layer, X)
    assert ei.value.name == "SLIM_ERR_WORKSPACE"
    Y = lib.linear_noalloc(layer, X[:496])
    torch.cuda.synchronize()
    assert np.all(from_dev_bf16(Y) == 0.0)
