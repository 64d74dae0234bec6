"""Pins for the oracle's quantization step (no GPU).

The oracle computes s = fp16(fp32(amax / 7)) and q = clip(rint(w / s), -7, 7)
with numpy's float32/float16 arithmetic.  These tests check it against an
independent exact-rational implementation of IEEE round-to-nearest-even and a
brute-force nearest-integer search, plus the hand-derived fixture and closed
forms (SLiM pipeline step 1: symmetric quantization, Fig. 7.1 caption;
4-bit with group 128, summary page).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from sparse_int4_linear_b200.workload import LayerSpec, make_layer
from exact_fp import f16, f32, nearest_q

HERE = os.path.dirname(os.path.abspath(__file__))


def _frac_f32(v):
    return Fraction(float(np.float32(v)))


def _bits_from_values(vals):
    a = np.asarray(vals, dtype=np.float32)
    bits = (a.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_bits_to_f32(bits), a), "fixture value is not exact bf16"
    return bits


def test_scale_matches_exact_rounding_random():
    li = make_layer(LayerSpec("t", 512, 24, 0, 11, 0.02, 0, 1.0), 1)
    W = oracle.bf16_bits_to_f32(li.W)
    q, s16 = oracle.quantize(W)
    for n in range(W.shape[0]):
        for g in range(W.shape[1] // 128):
            amax = max(abs(Fraction(float(v))) for v in W[n, g * 128:(g + 1) * 128])
            want = f16(f32(amax / 7))
            assert Fraction(float(s16[n, g])) == want


@pytest.mark.parametrize("amax", [1.0, 3.0, 0.02, 1e-3, 7 * 2.0 ** -7, 2.0 ** -20, 1e-9, 450000.0, 458752.0])
def test_scale_edge_values(amax):
    w = np.zeros((1, 128), dtype=np.float32)
    w[0, 5] = np.float32(amax)
    want = f16(f32(Fraction(float(np.float32(amax))) / 7))
    if want is None:
        with pytest.raises(oracle.OracleRangeError):
            oracle.quantize(w)
        return
    q, s16 = oracle.quantize(w)
    assert Fraction(float(s16[0, 0])) == want


def test_q_is_bruteforce_nearest():
    li = make_layer(LayerSpec("t", 256, 8, 0, 12, 0.02, 0, 1.0), 1)
    W = oracle.bf16_bits_to_f32(li.W)
    q, s16 = oracle.quantize(W)
    for n in range(W.shape[0]):
        for g in range(2):
            s = Fraction(float(s16[n, g]))
            for k in range(g * 128, (g + 1) * 128):
                assert int(q[n, k]) == nearest_q(Fraction(float(W[n, k])), s), (n, k)


def test_max_abs_q_is_seven_for_normal_scales():
    li = make_layer(LayerSpec("t", 1024, 64, 0, 13, 0.02, 0, 1.0), 1)
    q, s16 = oracle.quantize(oracle.bf16_bits_to_f32(li.W))
    gmax = np.abs(q.reshape(64, 8, 128)).max(axis=2)
    assert np.all(s16 > 0)
    assert np.all(gmax == 7)
    assert np.abs(q).max() <= 7


def test_symmetry_negating_w_negates_q():
    li = make_layer(LayerSpec("t", 256, 16, 0, 14, 0.02, 0, 1.0), 1)
    W = oracle.bf16_bits_to_f32(li.W)
    q1, s1 = oracle.quantize(W)
    q2, s2 = oracle.quantize(-W)
    assert np.array_equal(q1, -q2)
    assert np.array_equal(s1.view(np.uint16), s2.view(np.uint16))


def test_scale_uses_only_its_own_group():
    """Changing one group's values leaves every other group's q and scale unchanged."""
    li = make_layer(LayerSpec("t", 512, 4, 0, 15, 0.02, 0, 1.0), 1)
    W = oracle.bf16_bits_to_f32(li.W).copy()
    q1, s1 = oracle.quantize(W)
    W[:, 128:256] *= np.float32(8.0)
    q2, s2 = oracle.quantize(W)
    keep = np.r_[0:128, 256:512]
    assert np.array_equal(q1[:, keep], q2[:, keep])
    assert np.array_equal(s1[:, [0, 2, 3]], s2[:, [0, 2, 3]])
    assert not np.array_equal(s1[:, 1], s2[:, 1])


def test_nan_and_inf_raise():
    w = np.zeros((2, 128), dtype=np.float32)
    w[1, 3] = np.nan
    with pytest.raises(oracle.OracleRangeError):
        oracle.quantize(w)
    w[1, 3] = np.inf
    with pytest.raises(oracle.OracleRangeError):
        oracle.quantize(w)


def _fixture_rows():
    with open(os.path.join(HERE, "golden", "hand_example.json")) as f:
        fx = json.load(f)
    W = np.zeros((4, 128), dtype=np.float32)
    r0 = fx["rows"][0]["w_times_2pow7"]
    W[0, :len(r0)] = np.float32(r0) * np.float32(2.0 ** -7)
    r1 = fx["rows"][1]["w"]
    W[1, :len(r1)] = np.float32(r1)
    r3 = fx["rows"][3]["w_pow2"]
    W[3, :len(r3)] = np.float32([2.0 ** e for e in r3])
    return fx, W


def test_hand_example_quantization():
    fx, W = _fixture_rows()
    bits = _bits_from_values(W)
    q, s16 = oracle.quantize(oracle.bf16_bits_to_f32(bits))
    for n, row in enumerate(fx["rows"]):
        assert int(s16.view(np.uint16)[n, 0]) == int(row["scale_bits"], 16), n
        head = row["q_head"]
        assert q[n, :len(head)].tolist() == head, n
        assert not np.any(q[n, len(head):]), n
