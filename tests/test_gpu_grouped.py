"""Grouped layers: several compressed linears that read the same X packed
into one layer (for example the q, k and v projections of a decoder block,
or its gate and up projections) and computed by one call.

A grouped layer must give, row for row, what the separate linears give:
- its canonical bytes are the concatenation of the linears' canonical bytes,
  bit for bit (packing is row-local), and equal to the oracle's pack of the
  stacked weights;
- its output columns of linear g match the fp64 oracle of linear g alone
  (W_g, L_g, R_g) within the forward tolerance, on every path (single-launch
  decode, token-tiled decode, tensor-core prefill).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, oracle_reference, to_dev
from sparse_int4_linear_b200.workload import LayerSpec, make_layer

pytestmark = pytest.mark.gpu

SHAPES = [
    # K, row counts of the fused linears, r
    (512, (256, 256, 256), 32),       # q, k, v of equal width
    (1024, (512, 512), 16),           # gate, up
    (512, (1024, 256, 256), 64),      # q wider than k and v
    (256, (256, 40), 16),             # ragged last linear
    (384, (256, 256), 0),             # no adapter
    (256, (512, 1024, 40), 32),       # boundaries on 512 rows: the prefill CTA pairs serve it
]


def _members(K, Ns, r, M, seed):
    lis = [make_layer(LayerSpec(f"g{i}", K, n, r, seed + 17 * i, 0.02, max(1, K // 100), 20.0), M)
           for i, n in enumerate(Ns)]
    return lis, lis[0].X


def _pack(lib, lis, r):
    return lib.pack_grouped([to_dev(li.W) for li in lis],
                            [to_dev(li.L) for li in lis] if r else None,
                            [to_dev(li.R) for li in lis] if r else None)


@pytest.mark.parametrize("K,Ns,r", SHAPES)
def test_grouped_pack_is_the_concatenation(lib, K, Ns, r):
    lis, _ = _members(K, Ns, r, 1, 300 + K + r)
    layer = _pack(lib, lis, r)
    vals, meta, sc = (t.cpu().numpy() for t in layer.canonical())
    ref = oracle.pack_layer(np.concatenate([li.W for li in lis], 0))
    assert np.array_equal(vals, ref[0]) and np.array_equal(meta, ref[1])
    assert np.array_equal(sc.view(np.uint16), ref[2].view(np.uint16))
    row = 0
    for li, n in zip(lis, Ns):
        single = lib.pack(to_dev(li.W), to_dev(li.L) if r else None, to_dev(li.R) if r else None)
        sv, sm, ss = (t.cpu().numpy() for t in single.canonical())
        assert np.array_equal(vals[row:row + n], sv) and np.array_equal(meta[row:row + n], sm)
        assert np.array_equal(sc[row:row + n], ss)
        row += n


@pytest.mark.parametrize("M", [1, 5, 16, 33, 300])
@pytest.mark.parametrize("K,Ns,r", SHAPES)
def test_grouped_forward_matches_each_linear(lib, K, Ns, r, M):
    lis, X = _members(K, Ns, r, M, 700 + K + r)
    layer = _pack(lib, lis, r)
    Y = lib.linear(layer, to_dev(X))
    torch.cuda.synchronize()
    lib.sync_status(layer)
    Yh = from_dev_bf16(Y)
    row = 0
    for g, (li, n) in enumerate(zip(lis, Ns)):
        ref = oracle_reference(li, X)
        rel, mab = oracle.errors(Yh[:, row:row + n], ref)
        assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, \
            f"K={K} Ns={Ns} r={r} M={M} linear {g}: rel={rel:.3e} maxabs={mab:.3e}"
        row += n


def test_grouped_decode_is_one_launch(lib):
    """q, k, v of LLaMA-2-7B width fused: one kernel per decode call."""
    lis, X = _members(4096, (4096, 4096, 4096), 128, 4, 41)
    layer = _pack(lib, lis, 128)
    assert layer.launches(1) == 1 and layer.launches(4) == 1
    Y = lib.linear(layer, to_dev(X[:4]))
    torch.cuda.synchronize()
    lib.sync_status(layer)
    rows = np.array([0, 1, 2047, 4095])
    Yh = from_dev_bf16(Y)
    for g, li in enumerate(lis):
        ref = oracle_reference(li, X[:4], rows)
        rel, mab = oracle.errors(Yh[:, g * 4096 + rows], ref)
        assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, (g, rel, mab)
