"""Pins for the oracle's forward (no GPU).

Y = X W_eff^T + (X L) R: forward of a linear layer, thesis §2.1 (Y = X W^T,
W of shape d_out x d_in); the low-rank adapter is a separate path added to the
sparse product (§4, lazy low-rank adapters).  The pins use explicit loops
over the packed bytes on tiny shapes, the identity probe, linearity and the
r = 0 reduction.
"""
import numpy as np

import oracle
from sparse_int4_linear_b200.workload import LayerSpec, make_layer
from test_oracle_prune_pack import decode_bytes_loop


def _bits(a):
    a = np.asarray(a, dtype=np.float32)
    b = (a.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_bits_to_f32(b), a)
    return b


def _scales_f64(sc_bits):
    return sc_bits.view(np.float16).astype(np.float64)


def loop_forward(vals, meta, sc_bits, L, R, X):
    """Group-by-group sum over kept positions, then the adapter, in plain loops."""
    q = decode_bytes_loop(vals, meta)
    s = _scales_f64(sc_bits)
    x = oracle.bf16_bits_to_f64(X)
    N, K = q.shape
    M = x.shape[0]
    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for g in range(K // 128):
                part = 0.0
                for k in range(g * 128, (g + 1) * 128):
                    if q[n, k]:
                        part += float(q[n, k]) * x[m, k]
                tot += s[n, g] * part
            Y[m, n] = tot
    if L is not None:
        l = oracle.bf16_bits_to_f64(L)
        rr = oracle.bf16_bits_to_f64(R)
        r = l.shape[1]
        for m in range(M):
            t = [sum(x[m, k] * l[k, j] for k in range(K)) for j in range(r)]
            for n in range(N):
                Y[m, n] += sum(t[j] * rr[j, n] for j in range(r))
    return Y


def test_forward_matches_loops_tiny():
    li = make_layer(LayerSpec("t", 256, 6, 3, 31, 0.02, 2, 20.0), 3)
    vals, meta, sc = oracle.pack_layer(li.W)
    Y = oracle.forward(vals, meta, sc, li.L, li.R, li.X)
    Yl = loop_forward(vals, meta, sc, li.L, li.R, li.X)
    assert Y.shape == (3, 6)
    assert np.allclose(Y, Yl, rtol=1e-12, atol=1e-12)


def test_r0_is_sparse_quantized_matmul_only():
    li = make_layer(LayerSpec("t", 256, 5, 0, 32, 0.02, 2, 20.0), 2)
    vals, meta, sc = oracle.pack_layer(li.W)
    Y = oracle.forward(vals, meta, sc, None, None, li.X)
    assert np.allclose(Y, loop_forward(vals, meta, sc, None, None, li.X), rtol=1e-12, atol=1e-12)
    # and equals the full forward minus the adapter of a layer with r > 0
    li2 = make_layer(LayerSpec("t", 256, 5, 4, 32, 0.02, 2, 20.0), 2)
    v2, m2, s2 = oracle.pack_layer(li2.W)
    Yfull = oracle.forward(v2, m2, s2, li2.L, li2.R, li2.X)
    Y0 = oracle.forward(v2, m2, s2, None, None, li2.X)
    x = oracle.bf16_bits_to_f64(li2.X)
    l = oracle.bf16_bits_to_f64(li2.L)
    r = oracle.bf16_bits_to_f64(li2.R)
    ad = np.array([[sum(sum(x[m, k] * l[k, j] for k in range(256)) * r[j, n] for j in range(4))
                    for n in range(5)] for m in range(2)])
    assert np.allclose(Yfull - Y0, ad, rtol=1e-10, atol=1e-14)


def test_identity_probe_pins_orientation():
    """X = I_K returns W_eff^T + L R (rows = input channels, cols = outputs)."""
    K, N, r = 128, 7, 2
    li = make_layer(LayerSpec("t", K, N, r, 33, 0.02, 0, 1.0), 1)
    vals, meta, sc = oracle.pack_layer(li.W)
    X = _bits(np.eye(K, dtype=np.float32))
    Y = oracle.forward(vals, meta, sc, li.L, li.R, X)
    q = decode_bytes_loop(vals, meta).astype(np.float64)
    s = _scales_f64(sc)
    W_eff = q * s[:, [0]]
    LR = oracle.bf16_bits_to_f64(li.L) @ oracle.bf16_bits_to_f64(li.R)
    assert Y.shape == (K, N)
    for k in range(K):
        for n in range(N):
            assert abs(Y[k, n] - (W_eff[n, k] + LR[k, n])) <= 1e-15


def test_linearity_in_x():
    li = make_layer(LayerSpec("t", 256, 9, 4, 34, 0.02, 0, 1.0), 1)
    vals, meta, sc = oracle.pack_layer(li.W)
    rng = np.random.default_rng(3)
    X1 = rng.integers(-8, 9, size=(3, 256)).astype(np.float32)
    X2 = rng.integers(-8, 9, size=(3, 256)).astype(np.float32)
    f = lambda X: oracle.forward(vals, meta, sc, li.L, li.R, _bits(X))
    assert np.allclose(f(X1 + X2), f(X1) + f(X2), rtol=1e-12, atol=1e-12)
    assert np.allclose(f(3 * X1), 3 * f(X1), rtol=1e-12, atol=1e-12)


def test_transposed_weight_would_be_caught():
    """A square layer: using W_eff instead of W_eff^T changes the result."""
    li = make_layer(LayerSpec("t", 128, 128, 0, 35, 0.02, 0, 1.0), 2)
    vals, meta, sc = oracle.pack_layer(li.W)
    Y = oracle.forward(vals, meta, sc, None, None, li.X)
    W_eff = oracle.effective_weight(vals, meta, sc)
    x = oracle.bf16_bits_to_f64(li.X)
    assert np.allclose(Y, x @ W_eff.T)
    assert not np.allclose(Y, x @ W_eff)


def test_error_metrics():
    Yr = np.array([[1.0, -2.0], [3.0, 4.0]])
    assert oracle.errors(Yr, Yr) == (0.0, 0.0)
    Y = Yr.copy()
    Y[1, 1] += 0.02
    rel, mab = oracle.errors(Y, Yr)
    assert abs(rel - 0.02 / np.sqrt(30.0)) < 1e-15
    assert abs(mab - 0.005) < 1e-15
    assert oracle.within_tolerance(Y, Yr)
    Y[0, 0] += 0.5
    assert not oracle.within_tolerance(Y, Yr)


def test_adapter_down_identity_probe_and_loops():
    """T = X L (the adapter's first contraction, §4 lazy low-rank adapters):
    X = I_K returns L itself (pins the orientation: T is [M][r], L is [K][r]);
    on a non-square tiny case every element equals a plain loop over K."""
    K, r = 128, 3
    li = make_layer(LayerSpec("t", K, 4, r, 36, 0.02, 0, 1.0), 1)
    T_eye = oracle.adapter_down(li.L, _bits(np.eye(K, dtype=np.float32)))
    assert T_eye.shape == (K, r)
    assert np.array_equal(T_eye, oracle.bf16_bits_to_f64(li.L))
    li2 = make_layer(LayerSpec("t", 256, 4, 5, 37, 0.02, 3, 20.0), 2)
    T = oracle.adapter_down(li2.L, li2.X)
    x = oracle.bf16_bits_to_f64(li2.X)
    l = oracle.bf16_bits_to_f64(li2.L)
    assert T.shape == (2, 5)
    for m in range(2):
        for j in range(5):
            ref = 0.0
            for k in range(256):
                ref += x[m, k] * l[k, j]
            assert abs(T[m, j] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_adapter_term_is_adapter_down_times_r():
    """The forward's adapter term is exactly (X L) R with T = adapter_down(L, X)."""
    li = make_layer(LayerSpec("t", 384, 6, 4, 38, 0.02, 3, 20.0), 3)
    vals, meta, sc = oracle.pack_layer(li.W)
    diff = oracle.forward(vals, meta, sc, li.L, li.R, li.X) - oracle.forward(vals, meta, sc, None, None, li.X)
    T = oracle.adapter_down(li.L, li.X)
    assert np.allclose(diff, T @ oracle.bf16_bits_to_f64(li.R), rtol=1e-11, atol=1e-14)
