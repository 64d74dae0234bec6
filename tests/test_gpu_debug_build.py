"""The debug build (libslim_debug.so, SLIM_DEBUG: kernel index checks that
record SLIM_ERR_BOUNDS and skip the access) computes what the release build
computes: on every forward path its results match the fp64 oracle and no
check fires (the status word stays SLIM_OK).  The binding picks the library
at import, so the calls run in a child process with SLIM_LIBRARY=debug."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys
import numpy as np, torch
sys.path.insert(0, os.environ["SLIM_ROOT"]); sys.path.insert(0, os.path.join(os.environ["SLIM_ROOT"], "tests"))
import oracle
from gpu_util import to_dev, from_dev_bf16
from sparse_int4_linear_b200 import slim
from sparse_int4_linear_b200.workload import LayerSpec, make_layer
assert slim.LIB_PATH.endswith("libslim_debug.so"), slim.LIB_PATH
cases = [  # K, N, r, M, adapter bits, tuning
    (4096, 4096, 128, 1, 16, {}), (4096, 1024, 64, 16, 16, {}), (2048, 520, 20, 3, 16, {}),
    (1024, 600, 64, 7, 16, {"SLIM_NO_STREAM": "1"}), (1024, 600, 64, 40, 16, {"SLIM_NO_PREFILL": "1"}),
    (1024, 600, 64, 300, 16, {}), (1024, 2048, 64, 512, 16, {}), (4096, 4096, 128, 1, 4, {}),
    (1024, 600, 64, 300, 4, {}),
]
for K, N, r, M, bits, env in cases:
    for k in ("SLIM_NO_STREAM", "SLIM_NO_PREFILL"):
        os.environ.pop(k, None)
    os.environ.update(env)
    slim.tuning_reload()
    li = make_layer(LayerSpec("dbg", K, N, r, 900 + K % 97 + M, 0.02, max(1, K // 100), 20.0), M)
    layer = slim.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R), adapter_bits=bits)
    Y = from_dev_bf16(slim.linear(layer, to_dev(li.X)))
    slim.sync_status(layer)          # raises SlimError on SLIM_ERR_BOUNDS (or any device error)
    vals, meta, sc = oracle.pack_layer(li.W)
    fwd = oracle.forward_quantized_adapters if bits == 4 else oracle.forward
    rel, mab = oracle.errors(Y, fwd(vals, meta, sc, li.L, li.R, li.X))
    assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, (K, N, r, M, bits, env, rel, mab)
    print(f"debug ok K={K} N={N} r={r} M={M} bits={bits} {env} launches={layer.launches(M)} rel={rel:.2e}")
# the no-allocation entry point (its own scratch)
li = make_layer(LayerSpec("dbg", 2048, 512, 128, 950, 0.02, 20, 20.0), 40)
layer = slim.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
Y = from_dev_bf16(slim.linear_noalloc(layer, to_dev(li.X)))
slim.sync_status(layer)
vals, meta, sc = oracle.pack_layer(li.W)
rel, mab = oracle.errors(Y, oracle.forward(vals, meta, sc, li.L, li.R, li.X))
assert rel <= oracle.REL_FRO_TOL and mab <= oracle.MAX_ABS_TOL, (rel, mab)
print("debug ok noalloc")
'''


def test_debug_build_matches_oracle_without_check_failures():
    lib = os.path.join(ROOT, "sparse_int4_linear_b200", "libslim_debug.so")
    if not os.path.exists(lib):
        from sparse_int4_linear_b200 import build
        build.build(debug=True)
    env = dict(os.environ, SLIM_LIBRARY="debug", SLIM_ROOT=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert r.stdout.count("debug ok") == 10, r.stdout
