"""Every output element of full-size layers against the fp64 oracle.

The other full-size tests compare sampled output rows; here every row and
every token of the 7B MLP pair at its prefill batch (M = 2048: every
128-row weight-image tile, every 512-row CTA-pair block and every token tile
of the tensor-core path) and of the 70B q projection at a decode batch
(M = 16) and a prefill batch (M = 512) is compared.  Acceptance as in every
parity test: relative Frobenius error <= 5e-3 and max-abs error
<= 2e-2 * max|Y_ref| (Y = X W^T, thesis §2.1, plus the adapter path, §4).
"""
import pytest
import torch

import oracle
from gpu_util import from_dev_bf16, oracle_reference, to_dev
from sparse_int4_linear_b200.workload import CONFIGS, make_layer

pytestmark = pytest.mark.gpu

FULL = [
    (3, 0, 2048),   # 7B up 4096 -> 11008
    (3, 1, 2048),   # 7B down 11008 -> 4096
    (5, 0, 16),     # 70B q 8192 x 8192, decode
    (5, 0, 512),    # 70B q, prefill
]


@pytest.mark.parametrize("cfg,idx,M", FULL)
def test_every_output_element(lib, cfg, idx, M):
    spec = CONFIGS[cfg][0][idx]
    li = make_layer(spec, M)
    layer = lib.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    Y = lib.linear(layer, to_dev(li.X))
    torch.cuda.synchronize()
    lib.sync_status(layer)
    got = from_dev_bf16(Y)
    del Y, layer
    ref = oracle_reference(li, li.X)
    assert got.shape == ref.shape == (M, spec.N)
    rel, mab = oracle.errors(got, ref)
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, f"{spec.name} M={M}: rel={rel:.3e} maxabs={mab:.3e}"
