"""GPU parity of the single-launch decode path (M <= 16) in the cases its
work split treats specially: K cut into several panels (the X panel does not
fit shared memory), row tiles split across many warps and CTAs (their
segments meet in the workspace and the warp that completes a tile's arrival
count adds them), CTAs with idle warps (fewer chunks than warps), a ragged
last K block, the per-warp R^T prefetch, r = 0, the 15-warp CTAs of long
streams, and one workspace shared by a chain of layers of different adapter
ranks (the control block has to be ready for the next launch whatever used
it last).

Acceptance is the forward tolerance of every other parity test: relative
Frobenius error <= 5e-3 and max-abs error <= 2e-2 * max|Y_ref| against the
fp64 oracle (sampled output rows where the layer is large).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, oracle_reference, sample_rows, to_dev
from sparse_int4_linear_b200.workload import LayerSpec, make_layer

pytestmark = pytest.mark.gpu


def _check(Y, li, X, rows, what):
    got = from_dev_bf16(Y)
    if rows is not None:
        got = got[:, rows]
    rel, mab = oracle.errors(got, oracle_reference(li, X, rows))
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, f"{what}: rel={rel:.3e} maxabs={mab:.3e}"


CASES = [
    # K, N, r, M, sampled rows, kernels per call   (why)
    (32768, 64, 64, 8, None, 1),    # 10 K panels, each row tile split over ~66 warps; adapter X from global memory
    (24704, 96, 32, 8, None, 1),    # 7 panels and a half-filled last K block (K % 256 == 128)
    (16384, 32, 16, 9, None, 2),    # two token tiles on a short stream: the token-tiled pair
    (512, 11840, 256, 3, 64, 1),    # many row tiles, two K blocks each; R^T read through L2
    (8192, 40, 0, 16, None, 1),     # r = 0 with 4 panels (segments without an adapter)
    (1152, 4112, 48, 1, 64, 1),     # one token; the per-warp R^T prefetch
    (2048, 512, 64, 16, None, 1),   # two token tiles, two panels
    (16384, 4736, 32, 16, 64, 1),   # 15-warp CTAs, 4 panels
    (256, 64, 16, 3, None, 1),      # 4 chunks for a 7-warp CTA: idle warps
]


@pytest.mark.parametrize("K,N,r,M,nrows,launches", CASES)
def test_stream_work_split_cases(lib, K, N, r, M, nrows, launches):
    li = make_layer(LayerSpec("stream", K, N, r, 101 + K + N + r + M, 0.02, max(1, K // 100), 20.0), M)
    layer = lib.pack(to_dev(li.W), to_dev(li.L) if r else None, to_dev(li.R) if r else None)
    assert layer.launches(M) == launches
    X = to_dev(li.X)
    Y = lib.linear(layer, X)
    torch.cuda.synchronize()
    lib.sync_status(layer)
    rows = None if nrows is None else sample_rows(N, nrows, li.spec.seed)
    _check(Y, li, li.X, rows, f"K={K} N={N} r={r} M={M}")


# Layers of 2048 up to 64 chunks per SM with an adapter (70B k / v,
# 7B q_proj) run on the token-tiled pair at every M <= 16; with the warp
# count forced (8-warp CTAs, two adapter warps) the single-launch kernel
# still serves them.
@pytest.mark.parametrize("K,N,r,M", [(8192, 1024, 256, 1), (8192, 1024, 256, 4), (4096, 4096, 128, 1)])
def test_small_layers_pair_and_forced_single_launch(lib, tune, K, N, r, M):
    li = make_layer(LayerSpec("small", K, N, r, 301 + K + N + M, 0.02, K // 100, 20.0), M)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    rows = sample_rows(N, 96, li.spec.seed)
    X = to_dev(li.X)
    assert layer.launches(M) == 2
    Y = lib.linear(layer, X)
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _check(Y, li, li.X, rows, f"pair K={K} N={N} r={r} M={M}")
    tune(SLIM_STREAM_WARPS="8")
    assert layer.launches(M) == 1
    Y1 = lib.linear(layer, X)
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _check(Y1, li, li.X, rows, f"single launch K={K} N={N} r={r} M={M}")


def test_chain_of_layers_shares_one_workspace(lib):
    """Layers with r = 128, 256, 16, 0, 256 in a row, twice over, through one
    workspace (sized for the largest request) on one stream: every output
    must match its own oracle."""
    shapes = [(2048, 512, 128), (1024, 768, 256), (4096, 256, 16), (1024, 512, 0), (2048, 384, 256)]
    M = 7
    items = []
    for i, (K, N, r) in enumerate(shapes):
        li = make_layer(LayerSpec("chain", K, N, r, 500 + i, 0.02, max(1, K // 100), 20.0), M)
        layer = lib.pack(to_dev(li.W), to_dev(li.L) if r else None, to_dev(li.R) if r else None)
        items.append((li, layer, to_dev(li.X)))
    ws_bytes = max(layer.workspace_bytes(M) for _, layer, _ in items)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        for li, layer, X in items:
            outs.append((li, lib.linear(layer, X, ws=ws)))
    torch.cuda.synchronize()
    for li, layer, _ in items:
        lib.sync_status(layer)
    for li, Y in outs:
        s = li.spec
        _check(Y, li, li.X, None, f"chain K={s.K} N={s.N} r={s.r}")


def test_stream_repeated_calls_are_bit_identical(lib):
    li = make_layer(LayerSpec("rep", 8192, 320, 64, 77, 0.02, 81, 20.0), 16)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    X = to_dev(li.X)
    ws = lib.workspace(layer, 16)
    ys = [lib.linear(layer, X, ws=ws).clone() for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))
