"""Host planning of the forward, without a GPU: which kernels a call launches
and how much workspace it needs, from the library's own planner (its
148-SM default is the B200's count, so the plans are the ones a B200 gets).

The descriptors are filled by slim_layer_init / slim_grouped_layer_init,
which compute every field on the host and only then zero the device status
word; with no device that last step fails (SLIM_ERR_CUDA) and leaves a
complete descriptor, which the planning queries read without touching
device memory.  The buffer is a placeholder address, so the module is
skipped wherever a CUDA device is visible (the GPU tests cover the same
plans there, launching them).

Expectations: the launch counts asserted by the GPU tests for the same
shapes, the six LLaMA-2-70B-shaped linears and the 7B shapes of the bench,
the small-layer rule (layers of 2048 up to 64 chunks per SM with an adapter
take the token-tiled pair at every M <= 16 unless a warp count is forced),
and a workspace query that never decreases with M (a workspace sized for M
serves every M' <= M).
"""
import ctypes

import pytest
import torch

from sparse_int4_linear_b200 import slim

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="placeholder buffer: host-only planning checks run where no GPU is visible")

SLIM_OK, SLIM_ERR_CUDA = 0, -7
GROUP = 128


def _desc(K, Ns, r, bits=16):
    L = slim.SlimLayerDesc()
    n = (ctypes.c_int32 * len(Ns))(*Ns)
    nb = slim._lib.slim_grouped_layer_bytes(K, len(Ns), n, r, GROUP)
    assert nb > 0
    rc = slim._lib.slim_grouped_layer_init(ctypes.byref(L), K, len(Ns), n, r, GROUP, ctypes.c_void_p(1 << 30), nb,
                                           None)
    assert rc in (SLIM_OK, SLIM_ERR_CUDA) and L.magic != 0 and L.N == sum(Ns)
    if bits != 16:
        assert slim._lib.slim_layer_set_adapter_bits(ctypes.byref(L), bits) == SLIM_OK
    return L


def _launches(L, M):
    return slim._lib.slim_linear_launches(ctypes.byref(L), M)


def _ws(L, M):
    return slim._lib.slim_workspace_bytes(ctypes.byref(L), M)


@pytest.fixture
def warps(monkeypatch):
    """Force SLIM_STREAM_WARPS for one test (the library re-reads its tuning)."""
    def set_warps(v):
        monkeypatch.setenv("SLIM_STREAM_WARPS", v)
        slim._lib.slim_tuning_reload()
    yield set_warps
    monkeypatch.undo()
    slim._lib.slim_tuning_reload()


LLAMA70 = [("q", 8192, 8192), ("k", 8192, 1024), ("v", 8192, 1024), ("gate", 8192, 28672), ("up", 8192, 28672),
           ("down", 28672, 8192)]


@pytest.mark.parametrize("bits", [16, 4])
def test_llama70b_set(bits):
    lays = [_desc(K, [N], 256, bits) for _, K, N in LLAMA70]
    # one k_stream launch for q, gate, up, down; the token-tiled pair for k, v
    assert [_launches(L, 1) for L in lays] == [1, 2, 2, 1, 1, 1]
    assert [_launches(L, 16) for L in lays] == [1, 2, 2, 1, 1, 1]
    # prefill: T = X L, the weight images, the sparse MMA
    assert all(_launches(L, M) == 3 for L in lays for M in (17, 512, 4096))
    assert all(_launches(L, 0) == 0 for L in lays)


@pytest.mark.parametrize("K,N,r", [(8192, 1024, 256), (4096, 4096, 128)])
@pytest.mark.parametrize("bits", [16, 4])
def test_small_layer_rule_and_forced_single_launch(warps, K, N, r, bits):
    L = _desc(K, [N], r, bits)
    assert [_launches(L, M) for M in (1, 4, 8)] == [2, 2, 2]
    warps("8")
    assert [_launches(L, M) for M in (1, 4)] == [1, 1]


def test_llama7b_shapes():
    assert _launches(_desc(4096, [4096], 128), 1) == 2                 # q_proj: the pair
    qkv = _desc(4096, [4096, 4096, 4096], 128)                         # fused q, k, v: one stream
    assert _launches(qkv, 1) == 1 and _launches(qkv, 4) == 1
    assert _launches(_desc(4096, [11008], 128), 2048) == 3             # MLP up, prefill
    assert _launches(_desc(4096, [4096], 0), 1) == 1                   # no adapter: one launch


# (K, N, r, M, launches) as the GPU tests of the single-launch kernel assert them
STREAM_CASES = [
    (32768, 64, 64, 8, 1), (24704, 96, 32, 8, 1), (16384, 32, 16, 9, 2), (512, 11840, 256, 3, 1),
    (8192, 40, 0, 16, 1), (1152, 4112, 48, 1, 1), (2048, 512, 64, 16, 1), (16384, 4736, 32, 16, 1),
    (256, 64, 16, 3, 1), (16384, 4736, 32, 17, 3),
]


@pytest.mark.parametrize("K,N,r,M,n", STREAM_CASES)
def test_gpu_test_shapes(K, N, r, M, n):
    assert _launches(_desc(K, [N], r), M) == n


@pytest.mark.parametrize("K,Ns,r,bits", [(8192, [1024], 256, 16), (8192, [28672], 256, 16), (16384, [4736], 32, 16),
                                         (2048, [512], 64, 16), (32768, [64], 64, 16), (4096, [4096] * 3, 128, 16),
                                         (8192, [1024], 256, 4), (2048, [300], 136, 4)])
def test_workspace_never_decreases_with_M(K, Ns, r, bits):
    L = _desc(K, Ns, r, bits)
    Ms = list(range(0, 65)) + list(range(65, 1200, 7))
    ws = [_ws(L, M) for M in Ms]
    assert all(b >= a for a, b in zip(ws, ws[1:])), list(zip(Ms, ws))
    assert ws[0] == 0 and ws[-1] > 0
