"""One workspace across regimes, the token-tiled kernels at M > 16, and the
store-on-timeout rule.

* A workspace sized for M serves every call of up to M tokens, whatever path
  the previous call on it took: the tensor-core path (M > 16) and the
  token-tiled pair write their X·L where the single-launch kernel (M <= 16)
  keeps its row-tile arrival words and adapter partials.  Those words carry
  the launch's tag, so leftovers never count.  Checked on a layer whose
  single-launch plan splits K into several panels (arrival words in use),
  on the rows of the row tiles past 254.
* The token-tiled pair (adapter X·L, then the main product) at M > 16, when
  the tensor-core path is switched off, against the oracle; its X·L, read
  back from the workspace, against the oracle's adapter_down.
* When a wait of the single-launch kernel gives up, every output is written
  as zeros and SLIM_ERR_TIMEOUT is reported; the workspace stays usable.

Acceptance as in every parity test: relative Frobenius error <= 5e-3 and
max-abs error <= 2e-2 * max|Y_ref| against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, oracle_reference, sample_rows, to_dev
from sparse_int4_linear_b200.workload import LayerSpec, make_layer

pytestmark = pytest.mark.gpu


def _check(Y, li, X_bits, rows, what):
    got = from_dev_bf16(Y)
    if rows is not None:
        got = got[:, rows]
    rel, mab = oracle.errors(got, oracle_reference(li, X_bits, rows))
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, f"{what}: rel={rel:.3e} maxabs={mab:.3e}"


def _pack(lib, li):
    r = li.spec.r
    return lib.pack(to_dev(li.W), to_dev(li.L) if r else None, to_dev(li.R) if r else None)


def test_one_workspace_serves_every_regime(lib):
    K, N, r = 16384, 4736, 32
    li = make_layer(LayerSpec("regimes", K, N, r, 4242, 0.02, K // 100, 20.0), 300)
    layer = _pack(lib, li)
    assert layer.launches(16) == 1 and layer.launches(17) >= 2
    ws = torch.zeros(layer.workspace_bytes(300), dtype=torch.uint8, device="cuda")
    X = to_dev(li.X)
    # rows of the row tiles >= 254 (where earlier layouts collided), the edges, a sample
    rows = np.unique(np.concatenate([np.arange(254 * 16, N, 7), sample_rows(N, 32, 5)]))
    order = [17, 16, 300, 1, 16, 17, 16]
    outs = [(M, lib.linear(layer, X[:M], ws=ws).clone()) for M in order]
    torch.cuda.synchronize()
    lib.sync_status(layer)
    for M, Y in outs:
        _check(Y, li, li.X[:M], rows, f"M={M} after the sequence {order}")


@pytest.mark.parametrize("M", [17, 255, 1008])
def test_token_tiled_pair_at_large_M(lib, tune, M):
    tune(SLIM_NO_PREFILL="1")
    li = make_layer(LayerSpec("pair", 2048, 1536, 128, 77 + M, 0.02, 20, 20.0), M)
    layer = _pack(lib, li)
    assert layer.launches(M) == 2
    ws = lib.workspace(layer, M)
    Y = lib.linear(layer, to_dev(li.X), ws=ws)
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _check(Y, li, li.X, None, f"token-tiled pair M={M}")
    # T = X L sits after a 256-byte control block, bf16 [ceil(M/16)*16][r16]
    # row-major (the pair's workspace layout).
    r16 = 128
    T = ws[256:256 + ((M + 15) // 16) * 16 * r16 * 2].view(torch.bfloat16).view(-1, r16)[:M]
    rel, mab = oracle.errors(from_dev_bf16(T), oracle.adapter_down(li.L, li.X))
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, f"X L, M={M}: rel={rel:.3e} maxabs={mab:.3e}"


@pytest.mark.parametrize("K,N,r,M", [(2048, 512, 64, 16), (32768, 64, 64, 8), (16384, 4736, 32, 16)])
def test_single_launch_timeout_stores_zeros(lib, K, N, r, M):
    """One K panel, and several (where another CTA adds the row tile's panel
    partials and learns of the give-up from the row tile's arrival word), and
    16-warp CTAs with two token tiles."""
    li = make_layer(LayerSpec("timeout", K, N, r, 31 + K + M, 0.02, K // 100, 20.0), M)
    layer = _pack(lib, li)
    assert layer.launches(M) == 1
    ws = lib.workspace(layer, M)
    X = to_dev(li.X)
    Y = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    lib.test_stream_timeout(layer, X, ws, wait_us=2000, Y=Y)
    with pytest.raises(lib.SlimError) as err:
        lib.sync_status(layer)
    assert err.value.name == "SLIM_ERR_TIMEOUT"
    assert torch.count_nonzero(Y).item() == 0
    lib.sync_status(layer)                      # cleared by the read
    Y2 = lib.linear(layer, X, ws=ws)            # the same workspace, ready again
    torch.cuda.synchronize()
    lib.sync_status(layer)
    _check(Y2, li, li.X, None, "forward after a timed-out launch")
