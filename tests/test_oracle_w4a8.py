"""Pins for the oracle's W4A8 reading (no GPU; the CUDA path does not
implement 8-bit inputs).

The captions of Tables E.2 / E.5 name "4-bit weight and 8-bit input
quantization" and nothing more.  The oracle reads it as the weights'
symmetric abs-max rule at 8 bits with one fp32 scale per token, the integer
group sums of an int8 tensor core scaled by the weight group's fp16 scale and
the token's scale, and the adapter on the same dequantized input.  These
tests check the quantizer against exact-rational rounding and a brute-force
nearest integer to the fp32 quotient, its half-step error bound (a tie of the
fp32 quotient can cost one fp32 rounding more) and its grid identity, and the
integer-group forward against the dense float64 forward of the dequantized
operands (a different order of the same sums), so that a wrong group index,
a transposed scale or a dropped token scale fails.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact_fp import f32
from sparse_int4_linear_b200.workload import LayerSpec, make_layer


def f32_to_bf16_bits(x):
    """float32 values that are bf16-representable -> their bf16 bits."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "not bf16-representable"
    return (b >> 16).astype(np.uint16)


def nearest_q8(x: Fraction, s: Fraction) -> int:
    """Brute force: the q in [-127, 127] closest to the fp32-rounded quotient
    f32(x / s) (the reading divides in IEEE fp32, as the weights' quantizer
    does), ties to the even q."""
    t = f32(x / s)
    best = None
    for q in range(-127, 128):
        d = abs(t - q)
        if best is None or d < best[0] or (d == best[0] and q % 2 == 0):
            best = (d, q)
    return best[1]


def skewed_inputs(M, K, seed):
    """bf16 bits of X [M][K]: rows of very different magnitudes, one all-zero
    row, one row with a single non-zero, subnormal-range and large values."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)).astype(np.float32)
    X *= (10.0 ** rng.uniform(-6, 3, size=(M, 1))).astype(np.float32)
    X[1] = 0.0
    X[2] = 0.0
    X[2, K // 3] = -3.5
    bits = (X.view(np.uint32) >> 16).astype(np.uint16)   # truncate to bf16
    return bits


def test_quantizer_matches_exact_rounding():
    Xb = skewed_inputs(7, 96, 11)
    q, s = oracle.quantize_activations(Xb)
    X = oracle.bf16_bits_to_f32(Xb)
    assert q.dtype == np.int8 and q.shape == X.shape and s.shape == (7,)
    for m in range(X.shape[0]):
        amax = max(abs(Fraction(float(v))) for v in X[m])
        sc = f32(amax / 127)
        assert Fraction(float(s[m])) == sc, m
        for k in range(X.shape[1]):
            want = 0 if sc == 0 else nearest_q8(Fraction(float(X[m, k])), sc)
            assert int(q[m, k]) == want, (m, k)


def test_zero_row_and_single_value_row():
    Xb = skewed_inputs(4, 64, 3)
    q, s = oracle.quantize_activations(Xb)
    assert s[1] == 0 and not np.any(q[1])
    # one non-zero: it maps to +-127, every other entry of the row to 0
    assert q[2, 64 // 3] == -127 and np.count_nonzero(q[2]) == 1


def test_error_is_at_most_half_a_step():
    Xb = skewed_inputs(9, 256, 5)
    q, s = oracle.quantize_activations(Xb)
    X = oracle.bf16_bits_to_f64(Xb)
    err = np.abs(X - q.astype(np.float64) * s.astype(np.float64)[:, None])
    # half a step, plus the fp32 rounding of the quotient (at most 127 * 2^-24 steps)
    assert np.all(err <= (0.5 + 127 * 2.0 ** -24) * s.astype(np.float64)[:, None])
    assert np.all(np.abs(q) <= 127)


def test_identity_on_its_own_grid():
    """Rows q * 2^e with max |q| = 127: the scale is 2^e exactly and the
    quantized input equals the input, so W4A8 equals the plain forward."""
    rng = np.random.default_rng(8)
    M, K, N, r = 5, 256, 48, 16
    qx = rng.integers(-127, 128, size=(M, K))
    qx[:, 0] = 127
    e = rng.integers(-20, 4, size=(M, 1))
    X = (qx * np.exp2(e)).astype(np.float32)
    Xb = f32_to_bf16_bits(X)
    q, s = oracle.quantize_activations(Xb)
    assert np.array_equal(q, qx.astype(np.int8))
    assert np.array_equal(s, np.exp2(e[:, 0]).astype(np.float32))
    li = make_layer(LayerSpec("w4a8.grid", K, N, r, 21, 0.02, 3, 20.0), M)
    v, mt, sc = oracle.pack_layer(li.W)
    Y8 = oracle.forward_w4a8(v, mt, sc, li.L, li.R, Xb)
    Y = oracle.forward(v, mt, sc, li.L, li.R, Xb)
    assert np.max(np.abs(Y8 - Y)) <= 1e-12 * np.max(np.abs(Y))


@pytest.mark.parametrize("K,N,r,M", [(256, 40, 16, 3), (512, 96, 0, 5), (384, 33, 20, 1)])
def test_integer_groups_equal_the_dequantized_forward(K, N, r, M):
    li = make_layer(LayerSpec("w4a8", K, N, r, 40 + K + N + M, 0.02, 4, 20.0), M)
    v, mt, sc = oracle.pack_layer(li.W)
    Y8 = oracle.forward_w4a8(v, mt, sc, li.L if r else None, li.R if r else None, li.X)
    q, s = oracle.quantize_activations(li.X)
    Xh = q.astype(np.float64) * s.astype(np.float64)[:, None]
    ref = Xh @ oracle.effective_weight(v, mt, sc).T
    if r:
        ref = ref + (Xh @ oracle.bf16_bits_to_f64(li.L)) @ oracle.bf16_bits_to_f64(li.R)
    assert np.max(np.abs(Y8 - ref)) <= 1e-12 * np.max(np.abs(ref))
    # and 8-bit inputs stay close to the bf16-input forward (quantization error only)
    rel, _ = oracle.errors(Y8, oracle.forward(v, mt, sc, li.L if r else None, li.R if r else None, li.X))
    assert 0 < rel < 0.05


def test_nonfinite_input_is_a_range_error():
    Xb = skewed_inputs(3, 64, 9)
    Xb[0, 5] = 0x7F80   # +Inf
    with pytest.raises(oracle.OracleRangeError):
        oracle.quantize_activations(Xb)
