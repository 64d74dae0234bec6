"""GPU forward parity against the fp64 oracle.

Acceptance (the same for every shape and M): relative Frobenius error
<= 5e-3 and max-abs error <= 2e-2 * max|Y_ref|.  Forward Y = X W^T (thesis
§2.1) on the 2:4 int4 weight plus the separate adapter path (§4).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, oracle_reference, sample_rows, to_dev
from sparse_int4_linear_b200.workload import CONFIGS, LayerSpec, make_layer

pytestmark = pytest.mark.gpu


def _assert_close(Y, Y_ref, what):
    rel, mab = oracle.errors(Y, Y_ref)
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, f"{what}: rel={rel:.3e} maxabs={mab:.3e}"
    return rel, mab


def _run(lib, li, M, rows=None):
    spec = li.spec
    layer = lib.pack(to_dev(li.W), to_dev(li.L) if spec.r else None, to_dev(li.R) if spec.r else None)
    X = li.X[:M]
    Y = lib.linear(layer, to_dev(X))
    torch.cuda.synchronize()
    lib.sync_status(layer)
    Yh = from_dev_bf16(Y)
    ref = oracle_reference(li, X, rows)
    got = Yh if rows is None else Yh[:, rows]
    return _assert_close(got, ref, f"{spec.name} K={spec.K} N={spec.N} r={spec.r} M={M}")


@pytest.mark.parametrize("M", [16, 1, 5])
def test_config1_tiny(lib, M):
    li = make_layer(CONFIGS[1][0][0], 16)
    _run(lib, li, M)


RAGGED = [
    # K, N, r, M
    (128, 17, 7, 3), (384, 33, 0, 9), (640, 200, 16, 17), (128, 1, 1, 1), (1024, 48, 32, 33),
    (256, 256, 16, 255), (256, 130, 16, 257), (2304, 72, 48, 8), (512, 64, 0, 16), (768, 40, 24, 64),
]


@pytest.mark.parametrize("K,N,r,M", RAGGED)
def test_ragged_shapes(lib, K, N, r, M):
    li = make_layer(LayerSpec("rag", K, N, r, 7 + K + N + r + M, 0.02, max(1, K // 100), 20.0), M)
    _run(lib, li, M)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_config2_q_proj_full_oracle(lib, M):
    spec = CONFIGS[2][0][0]
    li = make_layer(spec, 16)
    _run(lib, li, M)


BIG = [(cfg, i, M) for cfg in (3, 4, 5) for i, s in enumerate(CONFIGS[cfg][0])
       for M in CONFIGS[cfg][1] if (cfg != 4 or s.name in ("7b.q", "7b.gate", "7b.down"))]


@pytest.mark.parametrize("cfg,idx,M", BIG)
def test_full_size_sampled_rows(lib, cfg, idx, M):
    spec = CONFIGS[cfg][0][idx]
    li = make_layer(spec, M)
    _run(lib, li, M, rows=sample_rows(spec.N, 64, spec.seed))


def test_empty_batch_is_noop(lib):
    li = make_layer(LayerSpec("t", 256, 64, 16, 3, 0.02, 0, 1.0), 1)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    Y = lib.linear(layer, X)
    assert Y.shape == (0, 64)


def test_deterministic_bits(lib):
    li = make_layer(LayerSpec("t", 4096, 512, 128, 4, 0.02, 41, 20.0), 16)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = to_dev(li.X)
    Y1 = lib.linear(layer, X).clone()
    Y2 = lib.linear(layer, X).clone()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_host_entry_point_matches_device(lib):
    li = make_layer(LayerSpec("t", 1024, 320, 16, 5, 0.02, 10, 20.0), 12)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    Yd = lib.linear(layer, to_dev(li.X)).cpu()
    Xh = torch.from_numpy(li.X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = lib.linear_host(layer, Xh)
    assert torch.equal(Yd.view(torch.int16), Yh.view(torch.int16))
    # Enqueued only: the result is there once the stream has passed the call.
    s = torch.cuda.Stream()
    Ya = torch.zeros(12, 320, dtype=torch.bfloat16).pin_memory()
    lib.linear_host(layer, Xh, Ya, stream=s, wait=False)
    s.synchronize()
    assert torch.equal(Yd.view(torch.int16), Ya.view(torch.int16))


def test_argument_errors_are_reported(lib):
    li = make_layer(LayerSpec("t", 256, 64, 16, 3, 0.02, 0, 1.0), 4)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = to_dev(li.X)
    ws = lib.workspace(layer, 4)
    with pytest.raises(lib.SlimError) as ei:                  # workspace too small
        lib.linear(layer, X, ws=ws[:16])
    assert ei.value.name == "SLIM_ERR_WORKSPACE"
    buf = torch.empty(4 * 256 * 2 + 2, dtype=torch.uint8, device="cuda")
    Xmis = buf[2:].view(torch.bfloat16).view(4, 256)          # 2-byte offset: misaligned
    with pytest.raises(lib.SlimError) as ei:
        lib.linear(layer, Xmis)
    assert ei.value.name == "SLIM_ERR_ALIGN"
    big = torch.empty(4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.SlimError) as ei:                  # Y overlaps X
        lib.linear(layer, big, Y=big[:, :64])
    assert ei.value.name == "SLIM_ERR_ARG"


@pytest.mark.parametrize("K,N,r,M", [(1024, 18944, 64, 384), (11008, 4096, 128, 2048)])
def test_prefill_tile_widths(lib, K, N, r, M):
    """The tensor-core path picks its tile by how the CTAs fill the SMs:
    74 blocks of 256 rows x 2 tiles of 192 tokens are one wave of 148 SMs
    exactly (one-SM CTAs; the CTA pair ties and the tie goes to them);
    8 blocks of 512 rows x 9 tiles of 240 tokens (144 CTAs of SM pairs) are
    one wave where 192 tokens would need two."""
    li = make_layer(LayerSpec("tiles", K, N, r, 9000 + N + M, 0.02, max(1, K // 100), 20.0), M)
    _run(lib, li, M, rows=sample_rows(N, 64, li.spec.seed))


@pytest.mark.parametrize("tile", ["2,192", "2,128", "1,128", "1,64", "pair,240", "pair,224", "pair,192", "pair,128"])
def test_prefill_every_cta_tile_shape(lib, tile, tune):
    """Every tensor-core tile the prefill path can pick (one CTA of 128-row
    halves x tokens, or a CTA pair of 512 rows x tokens on two SMs), forced in
    turn on one layer with a ragged token count and a ragged last row block."""
    tune(SLIM_PREFILL_TILE=tile)
    li = make_layer(LayerSpec("tile", 1152, 640, 48, 4242, 0.02, 11, 20.0), 300)
    _run(lib, li, 300)


@pytest.mark.parametrize("K,Ns,r", [(4096, [4096], 128), (4096, [11008], 128), (11008, [4096], 128),
                                    (1152, [640], 48), (256, [512, 1024, 40], 32), (2048, [512], 0)])
def test_workspace_query_covers_every_smaller_M(lib, K, Ns, r):
    """A caller sizes one workspace with slim_workspace_bytes(M) and uses it
    for every call of up to M tokens, so the query must never decrease with M:
    across the single-launch decode sizes, the switch to the tensor-core path,
    and its token tiles, whose width (and so the padding of T) changes with M."""
    layer = lib.PackedLayer(K, Ns if len(Ns) > 1 else Ns[0], r)
    ws = [layer.workspace_bytes(m) for m in range(1, 4097)]
    drops = [(m + 2, a, b) for m, (a, b) in enumerate(zip(ws, ws[1:])) if b < a]
    assert not drops, drops[:5]


def test_bounded_wait_gives_up_and_reports(lib):
    """The failure path of the kernels' waits: a wait on a barrier that
    nothing completes ends after its clock budget, leaves SLIM_ERR_TIMEOUT in
    the layer's status word (returned once, then cleared), and the context
    stays usable: the next forward on the same layer is correct."""
    li = make_layer(LayerSpec("timeout", 256, 256, 16, 77, 0.02, 2, 20.0), 4)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    lib.test_wait_timeout(layer, 2000)
    with pytest.raises(lib.SlimError) as err:
        lib.sync_status(layer)
    assert err.value.code == -6
    lib.sync_status(layer)                        # cleared by the read
    Y = lib.linear(layer, to_dev(li.X))
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _assert_close(from_dev_bf16(Y), oracle_reference(li, li.X), "forward after a timed-out wait")
