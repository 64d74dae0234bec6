"""GPU packing parity: slim_pack's canonical bytes are bit-identical to the
oracle's, and the decode-stream layout expands back to the same q and scales.

SLiM pipeline (Fig. 7.1 caption): symmetric quantization, then 2:4 pruning of
the quantized weights; 4-bit, group 128 (summary page); 2:4 along K with
packed values plus position metadata (§2.2.3).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import oracle_rows, sample_rows, to_dev
from sparse_int4_linear_b200.workload import CONFIGS, LayerSpec, make_layer

pytestmark = pytest.mark.gpu

SMALL = [(256, 256, 16), (128, 17, 7), (384, 33, 0), (640, 200, 16), (128, 1, 1), (1024, 48, 32)]


def _check_layer(lib, li, rows=None):
    spec = li.spec
    W = to_dev(li.W)
    L = to_dev(li.L) if spec.r else None
    R = to_dev(li.R) if spec.r else None
    layer = lib.pack(W, L, R)
    vals, meta, sc = layer.canonical()
    vals, meta, sc = vals.cpu().numpy(), meta.cpu().numpy(), sc.cpu().numpy().view(np.uint16)
    q_dec, sc_dec = lib.unpack_dec(layer)
    q_dec, sc_dec = q_dec.cpu().numpy(), sc_dec.cpu().numpy().view(np.uint16)
    if rows is None:
        rows = np.arange(spec.N)
    ov, om, os_ = oracle_rows(li.W, rows)
    assert np.array_equal(vals[rows], ov), "vals differ"
    assert np.array_equal(meta[rows], om), "meta differ"
    assert np.array_equal(sc[rows], os_), "scales differ"
    assert np.array_equal(q_dec[rows], oracle.unpack(ov, om)), "decode-stream q differs"
    assert np.array_equal(sc_dec[rows], os_), "decode-stream scales differ"
    return layer


@pytest.mark.parametrize("K,N,r", SMALL)
def test_pack_bit_exact_small(lib, K, N, r):
    li = make_layer(LayerSpec("t", K, N, r, 100 + K + N + r, 0.02, 0, 1.0), 1)
    _check_layer(lib, li)


def test_pack_bit_exact_tie_heavy(lib):
    """Integer-valued weights make |q| ties common (tie-break is part of the contract)."""
    rng = np.random.default_rng(5)
    W = rng.integers(-3, 4, size=(64, 512)).astype(np.float32) * np.float32(2.0 ** -5)
    bits = (W.view(np.uint32) >> 16).astype(np.uint16)
    li = make_layer(LayerSpec("t", 512, 64, 0, 6, 0.02, 0, 1.0), 1)
    li.W = bits
    _check_layer(lib, li)


def test_pack_bit_exact_edge_scales(lib):
    """All-zero rows, fp16-subnormal scales (where the clip is reached), mixed."""
    W = np.zeros((32, 256), dtype=np.float32)
    W[1, :5] = [2.0 ** -20, 2.0 ** -21, -2.0 ** -22, 0, 2.0 ** -24]
    W[2, :] = np.float32(1e-7) * np.arange(256, dtype=np.float32)
    W[3, 7] = 3.0
    W[4, 130] = -65000.0 * 7 / 8
    bits = (W.view(np.uint32) >> 16).astype(np.uint16)
    li = make_layer(LayerSpec("t", 256, 32, 0, 7, 0.02, 0, 1.0), 1)
    li.W = bits
    _check_layer(lib, li)


@pytest.mark.parametrize("bad", [np.nan, np.inf, 1.0e6])
def test_pack_range_error_sets_status(lib, bad):
    W = np.zeros((16, 256), dtype=np.float32)
    W[3, 9] = bad
    bits = (W.view(np.uint32) >> 16).astype(np.uint16)
    with pytest.raises(lib.SlimError) as ei:
        lib.pack(to_dev(bits))
    assert ei.value.name == "SLIM_ERR_RANGE"
    with pytest.raises(oracle.OracleRangeError):
        oracle.pack_layer(bits)


def test_pack_deterministic(lib):
    li = make_layer(LayerSpec("t", 1024, 96, 16, 9, 0.02, 0, 1.0), 1)
    a = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    b = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    ra, rb = a.regions(), b.regions()
    assert sorted(ra) == ["Lf", "Lp", "Rf", "Rp", "dec", "meta", "scales", "vals"]
    for k in ra:
        assert torch.equal(ra[k], rb[k]), k


FULL = sorted({(s.K, s.N, s.r, s.seed, s.sigma_w) for cfg in (2, 3, 5) for s in CONFIGS[cfg][0]})


@pytest.mark.parametrize("K,N,r,seed,sigma", FULL)
def test_pack_full_size_sampled_rows(lib, K, N, r, seed, sigma):
    li = make_layer(LayerSpec("full", K, N, r, seed, sigma, 0, 1.0), 1)
    _check_layer(lib, li, rows=sample_rows(N, 48, seed))
