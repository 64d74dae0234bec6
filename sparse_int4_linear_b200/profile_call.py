"""Run a few forward calls of one workload layer, for profilers.

    python -m sparse_int4_linear_b200.profile_call --cfg 5 --layer gate --M 1 --calls 4

Packs the seeded synthetic layer `--layer` of workload config `--cfg`
(sparse_int4_linear_b200.workload.CONFIGS), then issues `--calls` slim_linear
calls on one stream with one workspace, synchronises and checks the layer's
status word.  Nothing else runs on the GPU after packing, so a profiler can
skip the first calls (warm-up) and capture one launch of the kernel of
interest.  With `--graph` the calls are captured once as a CUDA graph and
replayed (the way the benchmark runs them).
"""
from __future__ import annotations

import argparse
import sys

import numpy as np
import torch

from sparse_int4_linear_b200 import slim
from sparse_int4_linear_b200.workload import CONFIGS, make_layer


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--cfg", type=int, default=5)
    ap.add_argument("--layer", default="gate", help="layer name within the config, e.g. q, k, gate, down")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--graph", action="store_true")
    a = ap.parse_args(argv)
    specs = [s for s in CONFIGS[a.cfg][0] if s.name.split(".")[-1] == a.layer]
    if not specs:
        print(f"no layer {a.layer!r} in config {a.cfg}", file=sys.stderr)
        return 2
    spec = specs[0]
    li = make_layer(spec, a.M)

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    layer = slim.pack(dev(li.W), dev(li.L) if spec.r else None, dev(li.R) if spec.r else None)
    X = dev(li.X)
    Y = torch.empty(a.M, spec.N, dtype=torch.bfloat16, device="cuda")
    ws = slim.workspace(layer, a.M)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    def calls():
        for _ in range(a.calls):
            slim.linear(layer, X, Y, ws, stream=stream)

    if a.graph:
        with torch.cuda.stream(stream):
            slim.linear(layer, X, Y, ws, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            calls()
        with torch.cuda.stream(stream):
            g.replay()
    else:
        calls()
    stream.synchronize()
    slim.sync_status(layer)
    print(f"{spec.name} K={spec.K} N={spec.N} r={spec.r} M={a.M}: {a.calls} calls, "
          f"{layer.launches(a.M)} launch(es) per call, ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
