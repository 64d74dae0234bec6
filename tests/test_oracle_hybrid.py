"""Pins for the oracle's hybrid dense / 2:4 tile reading (PATCH, Chapter 6
summary; no GPU: the CUDA path does not implement hybrid tiles).

Reading: 128 x 128 tiles, each dense or 2:4 by an input flag; the weights
are quantized first (SLiM step 1), then 2:4-pruned inside the 2:4 tiles
only.  Checked against: the SLiM effective weight when every tile is 2:4;
an exact-rational brute-force quantization when every tile is dense; tile
locality on a non-square tile grid with a ragged last row tile (a flag
broadcast along the wrong axis, or a tile of the wrong size, fails); the
2-of-4 count inside 2:4 tiles; and the identity probe X = I for the forward.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact_fp import f16, f32, nearest_q
from sparse_int4_linear_b200.workload import LayerSpec, make_layer


def _layer(N, K, r, M, seed):
    return make_layer(LayerSpec("hybrid", K, N, r, seed, 0.02, 4, 20.0), M)


def test_all_sparse_is_slim():
    li = _layer(300, 512, 16, 3, 1)
    flags = np.ones((3, 4), dtype=bool)
    v, m, s = oracle.pack_layer(li.W)
    assert np.array_equal(oracle.hybrid_effective_weight(li.W, flags), oracle.effective_weight(v, m, s))
    assert np.allclose(oracle.forward_hybrid(li.W, flags, li.L, li.R, li.X), oracle.forward(v, m, s, li.L, li.R, li.X),
                       rtol=0, atol=0)


def test_all_dense_is_exact_quantization():
    li = _layer(3, 256, 0, 1, 2)
    W = oracle.bf16_bits_to_f32(li.W)
    got = oracle.hybrid_effective_weight(li.W, np.zeros((1, 2), dtype=bool))
    for n in range(W.shape[0]):
        for g in range(W.shape[1] // 128):
            ks = range(g * 128, (g + 1) * 128)
            sc = f16(f32(max(abs(Fraction(float(W[n, k]))) for k in ks) / 7))
            for k in ks:
                want = 0 if sc == 0 else nearest_q(Fraction(float(W[n, k])), sc) * sc
                assert Fraction(float(got[n, k])) == want, (n, k)


def test_tiles_are_local():
    li = _layer(300, 512, 0, 1, 3)           # row tiles 128, 128, 44; four K tiles
    rng = np.random.default_rng(4)
    flags = rng.random((3, 4)) < 0.5
    flags[0, 0], flags[0, 1] = True, False   # both states present
    mixed = oracle.hybrid_effective_weight(li.W, flags)
    sparse = oracle.hybrid_effective_weight(li.W, np.ones((3, 4), dtype=bool))
    dense = oracle.hybrid_effective_weight(li.W, np.zeros((3, 4), dtype=bool))
    for tr in range(3):
        for tk in range(4):
            rows, cols = slice(tr * 128, min((tr + 1) * 128, 300)), slice(tk * 128, (tk + 1) * 128)
            want = sparse if flags[tr, tk] else dense
            assert np.array_equal(mixed[rows, cols], want[rows, cols]), (tr, tk)
    # inside 2:4 tiles at most two non-zeros per group of 4; dense tiles lose nothing
    nz = (mixed != 0).reshape(300, 128, 4).sum(axis=2)
    tile_of_group = np.repeat(np.repeat(flags, 128, axis=0)[:300], 32, axis=1)
    assert np.all(nz[tile_of_group] <= 2)
    assert np.array_equal(mixed[~np.repeat(np.repeat(flags, 128, axis=0)[:300], 128, axis=1)] != 0,
                          dense[~np.repeat(np.repeat(flags, 128, axis=0)[:300], 128, axis=1)] != 0)
    assert np.count_nonzero(dense) > np.count_nonzero(mixed) > np.count_nonzero(sparse)


def test_identity_probe_pins_the_transposition():
    li = _layer(40, 256, 0, 1, 5)
    flags = np.array([[True, False]])
    eye = (np.eye(256, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    Y = oracle.forward_hybrid(li.W, flags, None, None, eye)
    assert np.array_equal(Y, oracle.hybrid_effective_weight(li.W, flags).T)


def test_flag_grid_must_match():
    li = _layer(300, 512, 0, 1, 6)
    with pytest.raises(ValueError):
        oracle.hybrid_effective_weight(li.W, np.ones((4, 3), dtype=bool))
