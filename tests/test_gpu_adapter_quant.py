"""4-bit adapters ("Quantized SLiM": the low-rank adapters are quantized too,
thesis §7.4.3 "Low-rank adapter quantization", Tables E.13 / E.14 captions).

- The GPU's adapter quantization is bit-exact with the oracle's: q_L, s_L,
  q_R, s_R read back from the packed 4-bit layouts equal
  oracle.quantize_adapters, including R's short last group (r = 136), rank
  padding (r not a multiple of 16) and fused linears.
- The forward matches oracle.forward_quantized_adapters (fp64, X W_eff^T +
  (X L^) R^) within the forward tolerance on every path: the single-launch
  decode kernel (one and two adapter warps, one and several K panels), the
  token-tiled decode pair, the tensor-core prefill, grouped layers and the
  no-allocation entry point.
- The 4-bit forward is not the bf16 one: with the adapter's share of Y
  large, the bf16-adapter oracle is measurably further from it.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, sample_rows, to_dev
from sparse_int4_linear_b200.workload import LayerSpec, make_layer, n_outliers

pytestmark = pytest.mark.gpu


def _layer(K, N, r, M, seed, sigma_w=0.02):
    return make_layer(LayerSpec("aq", K, N, r, seed, sigma_w, n_outliers(K), 20.0), M)


def _pack4(lib, li):
    return lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R), adapter_bits=4)


def _ref(li, X_bits, rows=None):
    W = li.W if rows is None else li.W[rows]
    R = li.R if rows is None else li.R[:, rows]
    vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(W))
    return oracle.forward_quantized_adapters(vals, meta, sc, li.L, np.ascontiguousarray(R), X_bits)


def _check(Y, Y_ref, what):
    rel, mab = oracle.errors(Y, Y_ref)
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, (what, rel, mab)


@pytest.mark.parametrize("K,N,r", [(256, 40, 16), (512, 100, 136), (384, 33, 20), (8192, 1024, 256)])
def test_adapter_quantization_bit_exact(lib, K, N, r):
    li = _layer(K, N, r, 1, 700 + r)
    layer = _pack4(lib, li)
    assert layer.adapter_bits == 4
    qL, sL, qR, sR = (t.cpu().numpy() for t in lib.unpack_adapters(layer))
    rL, rsL, rR, rsR = oracle.quantize_adapters(li.L, li.R)
    assert np.array_equal(qL, rL) and np.array_equal(qR, rR)
    assert np.array_equal(sL.view(np.uint16), rsL.view(np.uint16))
    assert np.array_equal(sR.view(np.uint16), rsR.view(np.uint16))
    # the weights' packing is unaffected by the adapter format
    vals, meta, sc = (t.cpu().numpy() for t in layer.canonical())
    ref = oracle.pack_layer(li.W)
    assert np.array_equal(vals, ref[0]) and np.array_equal(meta, ref[1])


def test_grouped_adapter_quantization_bit_exact(lib):
    K, Ns, r = 256, (256, 40), 20
    lis = [_layer(K, n, r, 1, 720 + i) for i, n in enumerate(Ns)]
    layer = lib.pack_grouped([to_dev(li.W) for li in lis], [to_dev(li.L) for li in lis],
                             [to_dev(li.R) for li in lis], adapter_bits=4)
    qL, sL, qR, sR = (t.cpu().numpy() for t in lib.unpack_adapters(layer))
    L = np.concatenate([li.L for li in lis], 1)
    R = np.concatenate([li.R for li in lis], 1)
    rL, rsL, rR, rsR = oracle.quantize_adapters(L, R)
    assert np.array_equal(qL, rL) and np.array_equal(qR, rR)
    assert np.array_equal(sL.view(np.uint16), rsL.view(np.uint16))
    assert np.array_equal(sR.view(np.uint16), rsR.view(np.uint16))


def test_nonfinite_adapter_is_a_range_error(lib):
    li = _layer(256, 32, 16, 1, 730)
    L = li.L.copy()
    L[5, 3] = 0x7F80   # +Inf
    with pytest.raises(lib.SlimError) as e:
        lib.pack(to_dev(li.W), to_dev(L), to_dev(li.R), adapter_bits=4)
    assert e.value.name == "SLIM_ERR_RANGE"


# (K, N, r, M, launches per call, forced warps): 1 = the single-launch decode
# kernel, 2 = the token-tiled pair (the planner's choice for these shapes);
# with a forced warp count (SLIM_STREAM_WARPS) the single-launch kernel serves
# the 70B k / v and 7B q_proj shapes, which the planner sends to the pair.
STREAM_CASES = [
    (4096, 4096, 128, 1, 2, None),  # 7B q_proj: the pair
    (4096, 4096, 128, 1, 1, "8"),   # ... and the single-launch kernel
    (4096, 4096, 128, 16, 1, "8"),  # two K panels
    (8192, 1024, 256, 1, 2, None),  # 70B k / v: the pair
    (8192, 1024, 256, 1, 1, "8"),   # ... two adapter warps
    (8192, 1024, 256, 16, 2, None),  # token-tiled pair
    (28672, 512, 256, 16, 2, None),
    (2048, 300, 136, 5, 1, None),   # R's short group, ragged N
    (2048, 520, 20, 3, 1, None),    # rank padding
    (384, 33, 20, 3, 1, None),      # one CTA
    (512, 300, 136, 5, 2, None),
]


@pytest.mark.parametrize("K,N,r,M,nl,warps", STREAM_CASES)
def test_forward_decode_matches_oracle(lib, tune, K, N, r, M, nl, warps):
    if warps:
        tune(SLIM_STREAM_WARPS=warps)
    li = _layer(K, N, r, M, 740 + K % 997 + r + M, 0.015)
    layer = _pack4(lib, li)
    assert layer.launches(M) == nl
    Y = from_dev_bf16(lib.linear(layer, to_dev(li.X), ws=lib.workspace(layer, M)))
    lib.sync_status(layer)
    rows = sample_rows(N, 200, seed=K + M)
    _check(Y[:, rows], _ref(li, li.X, rows), ("decode", K, N, r, M))


@pytest.mark.parametrize("env,M", [({"SLIM_NO_STREAM": "1"}, 7), ({"SLIM_NO_PREFILL": "1"}, 40), ({}, 300),
                                   ({}, 512)])
def test_forward_other_paths_match_oracle(lib, tune, env, M):
    tune(**env)
    K, N, r = 1024, 600, 64
    li = _layer(K, N, r, M, 760 + M)
    layer = _pack4(lib, li)
    Y = from_dev_bf16(lib.linear(layer, to_dev(li.X), ws=lib.workspace(layer, M)))
    lib.sync_status(layer)
    _check(Y, _ref(li, li.X), (env, M))


@pytest.mark.parametrize("M", [1, 16, 300])
def test_grouped_forward_matches_oracle(lib, M):
    K, Ns, r = 512, (256, 256, 40), 32
    lis = [_layer(K, n, r, M, 780 + i) for i, n in enumerate(Ns)]
    X = lis[0].X
    layer = lib.pack_grouped([to_dev(li.W) for li in lis], [to_dev(li.L) for li in lis],
                             [to_dev(li.R) for li in lis], adapter_bits=4)
    Y = from_dev_bf16(lib.linear(layer, to_dev(X), ws=lib.workspace(layer, M)))
    lib.sync_status(layer)
    c = 0
    for li, n in zip(lis, Ns):
        _check(Y[:, c:c + n], _ref(li, X), ("grouped", M, n))
        c += n


@pytest.mark.parametrize("M", [1, 40])
def test_noalloc_matches_oracle(lib, M):
    K, N, r = 2048, 512, 128
    li = _layer(K, N, r, M, 800 + M)
    layer = _pack4(lib, li)
    Y = from_dev_bf16(lib.linear_noalloc(layer, to_dev(li.X)))
    lib.sync_status(layer)
    _check(Y, _ref(li, li.X), ("noalloc", M))


def test_four_bit_forward_differs_from_bf16_adapter(lib):
    """With the adapter a large share of Y (small W, large L, R), the 4-bit
    forward is within tolerance of the 4-bit oracle and measurably away from
    the bf16-adapter oracle, so the kernels really use the 4-bit factors."""
    K, N, r, M = 1024, 256, 64, 4
    li = make_layer(LayerSpec("aq", K, N, r, 820, 0.0005, 0, 1.0), M)
    scale = lambda bits, f: (np.ascontiguousarray(oracle.bf16_bits_to_f32(bits) * np.float32(f))
                             .view(np.uint32) >> 16).astype(np.uint16)
    L, R = scale(li.L, 8.0), scale(li.R, 8.0)       # powers of two: still exact bf16
    li = type(li)(li.spec, li.W, L, R, li.X)
    layer = _pack4(lib, li)
    Y = from_dev_bf16(lib.linear(layer, to_dev(li.X), ws=lib.workspace(layer, M)))
    lib.sync_status(layer)
    vals, meta, sc = oracle.pack_layer(li.W)
    Y4 = oracle.forward_quantized_adapters(vals, meta, sc, L, R, li.X)
    Y16 = oracle.forward(vals, meta, sc, L, R, li.X)
    rel4, _ = oracle.errors(Y, Y4)
    rel16, _ = oracle.errors(Y, Y16)
    assert rel4 <= oracle.REL_FRO_TOL
    assert rel16 > 4 * rel4, (rel4, rel16)
