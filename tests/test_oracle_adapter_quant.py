"""Pins for the oracle's adapter quantization (no GPU).

Quantized SLiM quantizes the low-rank adapters too (thesis §7.4.3 "Low-rank
adapter quantization"; Tables E.13 / E.14 captions).  The oracle's reading:
the weights' symmetric 4-bit abs-max quantizer with fp16 scales, in groups
of 128 along each factor's reduction dimension (K for L [K][r], r for
R [r][N], the last group of R shorter when r % 128 != 0).  These tests check
it against exact-rational rounding and a brute-force nearest q written out
per (column, group), closed forms, and a loop forward.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact_fp import f16, f32, nearest_q
from sparse_int4_linear_b200.workload import LayerSpec, make_layer


def brute_factor(F, group=128):
    """Exact per-(column, group) scales and q of a factor F [n_red][cols],
    groups running down each column (the reduction dimension)."""
    n_red, cols = F.shape
    ng = -(-n_red // group)
    q = np.zeros((n_red, cols), dtype=np.int64)
    s = [[None] * cols for _ in range(ng)]
    for c in range(cols):
        for gi in range(ng):
            rows = range(gi * group, min((gi + 1) * group, n_red))
            amax = max(abs(Fraction(float(F[i, c]))) for i in rows)
            sc = f16(f32(amax / 7))
            s[gi][c] = sc
            for i in rows:
                q[i, c] = 0 if sc == 0 else nearest_q(Fraction(float(F[i, c])), sc)
    return q, s


def skewed_factors(K, N, r, seed):
    """L, R bf16 bits whose columns (and R's short last group) differ in
    magnitude by powers of two, so a grouping along the wrong axis, or a
    short group merged with its neighbour, changes the scales."""
    li = make_layer(LayerSpec("aq", K, N, r, seed), 1)
    L = oracle.bf16_bits_to_f32(li.L).copy()
    R = oracle.bf16_bits_to_f32(li.R).copy()
    L *= (2.0 ** (np.arange(r) % 5)).astype(np.float32)[None, :]
    L[:128] *= np.float32(4.0)                      # the two K groups of a column differ
    R *= (2.0 ** (np.arange(N) % 3)).astype(np.float32)[None, :]
    R[128:] *= np.float32(16.0)                     # the short group of R (r > 128)
    to_bits = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    Lb, Rb = to_bits(L), to_bits(R)
    assert np.array_equal(oracle.bf16_bits_to_f32(Lb), L) and np.array_equal(oracle.bf16_bits_to_f32(Rb), R)
    return Lb, Rb, li.X


def test_shapes_and_ranges():
    Lb, Rb, _ = skewed_factors(256, 6, 136, 31)
    qL, sL, qR, sR = oracle.quantize_adapters(Lb, Rb)
    assert qL.shape == (256, 136) and sL.shape == (2, 136)
    assert qR.shape == (136, 6) and sR.shape == (2, 6)
    assert sL.dtype == np.float16 and sR.dtype == np.float16
    assert np.abs(qL).max() <= 7 and np.abs(qR).max() <= 7


def test_L_matches_bruteforce_groups_along_K():
    Lb, Rb, _ = skewed_factors(256, 6, 136, 32)
    qL, sL, _, _ = oracle.quantize_adapters(Lb, Rb)
    cols = list(range(0, 136, 7))          # every 7th column: all five magnitudes, both K groups
    Lf = oracle.bf16_bits_to_f32(Lb)[:, cols]
    qb, sb = brute_factor(Lf)
    assert np.array_equal(qL[:, cols].astype(np.int64), qb)
    for gi in range(2):
        for ci, c in enumerate(cols):
            assert Fraction(float(sL[gi, c])) == sb[gi][ci], (gi, c)


def test_R_matches_bruteforce_with_short_last_group():
    Lb, Rb, _ = skewed_factors(256, 6, 136, 33)
    _, _, qR, sR = oracle.quantize_adapters(Lb, Rb)
    Rf = oracle.bf16_bits_to_f32(Rb)
    qb, sb = brute_factor(Rf)               # groups [0, 128) and [128, 136) of each column
    assert np.array_equal(qR.astype(np.int64), qb)
    for gi in range(2):
        for n in range(6):
            assert Fraction(float(sR[gi, n])) == sb[gi][n], (gi, n)


def test_rank_below_group_is_one_group():
    li = make_layer(LayerSpec("aq", 128, 40, 16, 34), 1)
    _, _, qR, sR = oracle.quantize_adapters(li.L, li.R)
    Rf = oracle.bf16_bits_to_f32(li.R)
    assert sR.shape == (1, 40)
    qb, sb = brute_factor(Rf)
    assert np.array_equal(qR.astype(np.int64), qb)
    assert all(Fraction(float(sR[0, n])) == sb[0][n] for n in range(40))


def test_dequantization_error_is_at_most_half_a_step():
    Lb, Rb, _ = skewed_factors(256, 6, 136, 35)
    qL, sL, qR, sR = oracle.quantize_adapters(Lb, Rb)
    for F, q, s in ((oracle.bf16_bits_to_f64(Lb), qL, sL), (oracle.bf16_bits_to_f64(Rb), qR, sR)):
        Fh = oracle.dequantize_adapter(q, s)
        step = np.repeat(s.astype(np.float64), 128, axis=0)[: F.shape[0]]
        # |F| <= amax <= 7 s (1 + 2^-11): within half a step except past the
        # clip, where the excess is at most amax * 2^-11.
        assert np.all(np.abs(F - Fh) <= 0.5 * step + np.abs(F) * 2.0 ** -10)


def test_quantizer_is_identity_on_its_own_grid():
    """Factors whose every group already is q * s with max |q| = 7 and s a
    power of two come back unchanged, so the forward equals forward()."""
    rng = np.random.default_rng(36)
    K, N, r, M = 256, 24, 20, 3
    def grid(n_red, cols, exps):
        q = rng.integers(-7, 8, size=(n_red, cols))
        for c in range(cols):
            for g0 in range(0, n_red, 128):
                q[g0 + rng.integers(0, min(128, n_red - g0)), c] = 7 * rng.choice([-1, 1])
        s = np.array([[2.0 ** exps[(g0 // 128 + c) % len(exps)] for c in range(cols)] for g0 in range(0, n_red, 128)])
        F = (q * np.repeat(s, 128, axis=0)[:n_red]).astype(np.float32)
        return (F.view(np.uint32) >> 16).astype(np.uint16), q, s
    Lb, qL0, sL0 = grid(K, r, [-9, -7, -12])
    Rb, qR0, sR0 = grid(r, N, [-8, -10])
    qL, sL, qR, sR = oracle.quantize_adapters(Lb, Rb)
    assert np.array_equal(qL, qL0) and np.array_equal(qR, qR0)
    assert np.array_equal(sL.astype(np.float64), sL0) and np.array_equal(sR.astype(np.float64), sR0)
    li = make_layer(LayerSpec("aq", K, N, r, 37), M)
    vals, meta, sc = oracle.pack_layer(li.W)
    Y0 = oracle.forward(vals, meta, sc, Lb, Rb, li.X)
    Y1 = oracle.forward_quantized_adapters(vals, meta, sc, Lb, Rb, li.X)
    assert np.array_equal(Y0, Y1)


def test_forward_against_loops():
    K, N, r, M = 256, 10, 20, 3
    li = make_layer(LayerSpec("aq", K, N, r, 38), M)
    vals, meta, sc = oracle.pack_layer(li.W)
    Y = oracle.forward_quantized_adapters(vals, meta, sc, li.L, li.R, li.X)
    W_eff = oracle.effective_weight(vals, meta, sc)
    X = oracle.bf16_bits_to_f64(li.X)
    qL, sL = brute_factor(oracle.bf16_bits_to_f32(li.L))
    qR, sR = brute_factor(oracle.bf16_bits_to_f32(li.R))
    Lh = [[float(qL[k, j] * sL[k // 128][j]) for j in range(r)] for k in range(K)]
    Rh = [[float(qR[j, n] * sR[j // 128][n]) for n in range(N)] for j in range(r)]
    for m in range(M):
        T = [sum(X[m, k] * Lh[k][j] for k in range(K)) for j in range(r)]
        for n in range(N):
            y = sum(X[m, k] * W_eff[n, k] for k in range(K)) + sum(T[j] * Rh[j][n] for j in range(r))
            assert Y[m, n] == pytest.approx(y, rel=1e-12, abs=1e-12)


def test_no_adapter_is_the_plain_forward():
    li = make_layer(LayerSpec("aq", 256, 16, 0, 39), 2)
    vals, meta, sc = oracle.pack_layer(li.W)
    assert np.array_equal(oracle.forward_quantized_adapters(vals, meta, sc, None, None, li.X),
                          oracle.forward(vals, meta, sc, None, None, li.X))


def test_grouped_factors_quantize_per_column():
    """Side-by-side factors of fused linears (L [K][G r], R [r][sum N]) give
    each linear's own quantization: columns never share a group."""
    li = make_layer(LayerSpec("aq", 256, 48, 32, 40), 1)
    qL, sL, qR, sR = oracle.quantize_adapters(li.L, li.R)
    for c0, c1 in ((0, 16), (16, 32)):
        a = oracle.quantize_adapters(li.L[:, c0:c1], li.R[c0:c1, :])
        assert np.array_equal(a[0], qL[:, c0:c1]) and np.array_equal(a[1], sL[:, c0:c1])
    for n0, n1 in ((0, 20), (20, 48)):
        b = oracle.quantize_adapters(li.L, li.R[:, n0:n1])
        assert np.array_equal(b[2], qR[:, n0:n1]) and np.array_equal(b[3], sR[:, n0:n1])


def test_nonfinite_scale_is_a_range_error():
    L = np.zeros((128, 16), dtype=np.uint16)
    L[3, 2] = 0x7F80   # +Inf
    R = np.zeros((16, 8), dtype=np.uint16)
    with pytest.raises(oracle.OracleRangeError):
        oracle.quantize_adapters(L, R)
