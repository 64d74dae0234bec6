"""Pins for the oracle's 2:4 pruning and packing (no GPU).

2:4 structure along the reduction dimension with packed values and position
metadata: thesis §2.2.3 "Sparse Tensor Core Acceleration"; pruning applies
to the quantized weights: SLiM pipeline, Fig. 7.1 caption.
"""
import itertools
import json
import os

import numpy as np

import oracle
from sparse_int4_linear_b200.workload import LayerSpec, make_layer

HERE = os.path.dirname(os.path.abspath(__file__))


def brute_pairs(q):
    """Exhaustive search over all 6 two-of-four patterns, group by group."""
    N, K = q.shape
    out0 = np.zeros((N, K // 4), np.int8)
    out1 = np.zeros((N, K // 4), np.int8)
    for n in range(N):
        for c in range(K // 4):
            a = [abs(int(v)) for v in q[n, 4 * c:4 * c + 4]]
            best = None
            for (i, j) in itertools.combinations(range(4), 2):   # lexicographic order
                sc = a[i] + a[j]
                if best is None or sc > best[0]:
                    best = (sc, i, j)
            out0[n, c], out1[n, c] = best[1], best[2]
    return out0, out1


def stable_sort_pairs(q):
    """Equivalent reading: stable sort by -|q|, keep the first two, order them."""
    N, K = q.shape
    a = -np.abs(q.reshape(N, K // 4, 4).astype(np.int32))
    order = np.argsort(a, axis=-1, kind="stable")[..., :2]
    return np.min(order, -1).astype(np.int8), np.max(order, -1).astype(np.int8)


def _rand_q(N, K, seed, lo=-7, hi=7):
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=(N, K)).astype(np.int8)


def test_prune_matches_bruteforce_random_and_tie_heavy():
    for seed, (lo, hi) in enumerate([(-7, 7), (-1, 1), (0, 0), (-2, 2)]):
        q = _rand_q(16, 128, seed, lo, hi)
        i0, i1 = oracle.prune_2of4(q)
        b0, b1 = brute_pairs(q)
        assert np.array_equal(i0, b0) and np.array_equal(i1, b1)
        s0, s1 = stable_sort_pairs(q)
        assert np.array_equal(i0, s0) and np.array_equal(i1, s1)


def test_prune_invariants():
    li = make_layer(LayerSpec("t", 512, 32, 0, 21, 0.02, 0, 1.0), 1)
    q, _ = oracle.quantize(oracle.bf16_bits_to_f32(li.W))
    i0, i1 = oracle.prune_2of4(q)
    assert np.all(i0 < i1) and np.all(i0 >= 0) and np.all(i1 <= 3)
    m = oracle.mask_from_pairs(i0, i1)
    assert np.all(m.reshape(32, -1, 4).sum(-1) == 2)          # exactly 2 kept slots
    a = np.abs(q.reshape(32, -1, 4).astype(int))
    mk = m.reshape(32, -1, 4)
    kept_min = np.where(mk, a, 99).min(-1)
    drop_max = np.where(~mk, a, -1).max(-1)
    assert np.all(drop_max <= kept_min)                          # dropped never beat kept
    nnz = (np.where(mk, q.reshape(32, -1, 4), 0) != 0).sum(-1)
    assert np.all(nnz <= 2)


def decode_bytes_loop(vals, meta):
    """Byte-by-byte decoder written from the format description (no numpy tricks)."""
    N, G4 = vals.shape
    out = [[0] * (4 * G4) for _ in range(N)]
    for n in range(N):
        for c in range(G4):
            b = int(vals[n, c])
            lo, hi = b & 15, b >> 4
            v0 = lo - 16 if lo & 8 else lo
            v1 = hi - 16 if hi & 8 else hi
            mb = int(meta[n, c // 2])
            nib = (mb >> 4) if (c % 2) else (mb & 15)
            i0, i1 = nib & 3, nib >> 2
            out[n][4 * c + i0] = v0
            out[n][4 * c + i1] = v1
    return np.array(out, dtype=np.int8)


def test_pack_unpack_identity_and_loop_decoder():
    q = _rand_q(8, 256, 7)
    i0, i1 = oracle.prune_2of4(q)
    vals, meta = oracle.pack(q, i0, i1)
    assert vals.shape == (8, 64) and meta.shape == (8, 32)
    kept = np.where(oracle.mask_from_pairs(i0, i1), q, 0)
    assert np.array_equal(oracle.unpack(vals, meta), kept)
    assert np.array_equal(decode_bytes_loop(vals, meta), kept)


def test_pack_byte_sizes():
    for (N, K) in [(256, 256), (4096, 4096), (1024, 8192)]:
        assert oracle.canonical_bytes(N, K) == N * K * 3 // 8 + 2 * N * K // 128
    li = make_layer(LayerSpec("t", 256, 256, 0, 0, 0.02, 0, 1.0), 1)
    vals, meta, sc = oracle.pack_layer(li.W)
    assert vals.nbytes + meta.nbytes + sc.nbytes == oracle.canonical_bytes(256, 256)


def test_hand_example_bytes():
    with open(os.path.join(HERE, "golden", "hand_example.json")) as f:
        fx = json.load(f)
    from test_oracle_quant import _fixture_rows, _bits_from_values
    _, W = _fixture_rows()
    vals, meta, sc = oracle.pack_layer(_bits_from_values(W))
    q = oracle.unpack(vals, meta)
    for n, row in enumerate(fx["rows"]):
        vh = [int(x, 16) for x in row["vals_head"]]
        mh = [int(x, 16) for x in row["meta_head"]]
        assert vals[n, :len(vh)].tolist() == vh, n
        assert np.all(vals[n, len(vh):] == 0), n
        assert meta[n, :len(mh)].tolist() == mh, n
        assert np.all(meta[n, len(mh):] == 0x44), n
        assert int(sc[n, 0]) == int(row["scale_bits"], 16)
        i0, i1 = oracle.prune_2of4(oracle.quantize(oracle.bf16_bits_to_f32(_bits_from_values(W)))[0])
        assert [[int(a), int(b)] for a, b in zip(i0[n, :len(row["pairs_head"])], i1[n])] == row["pairs_head"]
    # the kept values of row 0 after pruning
    assert q[0, :20].tolist() == [7, -3, 0, 0, -2, 2, 0, 0, 1, -1, 0, 0, 0, 0, -2, 2, 0, 3, -3, 0]
