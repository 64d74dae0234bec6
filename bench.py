#!/usr/bin/env python3
"""Benchmark of the compressed linear layer on B200.

Workload: the LLaMA-2-7B q_proj shape (K = N = 4096), int4 2:4 weights with
group-128 fp16 scales and an r = 128 bf16 adapter, decode batches of
M = 1, 4 and 16 tokens; synthetic seeded inputs.

One step = every M of the sweep pushed through a stack of `--layers`
independently packed copies of that layer (M-major, so a layer's weights are
read again only after all the other copies have been read: with the default
60 copies, ~0.5 GB in between, four times the 126 MB L2, so every call reads
its weights from HBM).  The step is captured once as a CUDA graph and
replayed.  The metric is algorithmic bytes moved per second (GB/s): packed
values + metadata + scales + L + R + X + Y of every call.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl slim|reference]

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas, no collective on the data path); the whole-job value
is the sum of the ranks' bytes over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_int4_linear_b200.workload import CONFIGS, make_layer  # noqa: E402

M_SWEEP = (1, 4, 16)
SPEC = CONFIGS[2][0][0]   # 7B q_proj: K = N = 4096, r = 128
METRIC = "2:4+INT4+low-rank linear: GB/s (M≤16), TFLOP/s (M≥256) vs B200 roofline"
WORKLOAD = "LLaMA-2-7B q_proj K=N=4096, g=128 int4 + 2:4, adapter r=128 bf16, decode M in {1,4,16}"


def algorithmic_bytes(K, N, r, M):
    """vals + meta + scales + L + R + X + Y (the T = X L scratch excluded)."""
    return N * K // 4 + N * K // 8 + N * (K // 128) * 2 + 2 * K * r + 2 * r * N + 2 * M * K + 2 * M * N


def kept_flops(K, N, r, M):
    return 2 * M * N * (K // 2) + 2 * M * r * (K + N)


# DRAM bytes (read + write) of one launch of the single-launch decode kernel for
# the M = 1 call of this workload, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum).  None once the kernel has
# changed since that capture.
TRAFFIC_M1_LAUNCH = 8.72e6


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- distributed
def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:   # host-only runs of the rank plumbing (CPU tests)
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU baseline
def cpu_baseline(budget_s: float = 12.0):
    """The oracle forward as it stands, timed on the host cores on a bounded
    sample: repeated decode calls of the same workload until ~budget_s."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    li = make_layer(SPEC, max(M_SWEEP))
    vals, meta, sc = oracle.pack_layer(li.W)
    nbytes, calls = 0, 0
    t0 = time.perf_counter()
    while True:
        for M in M_SWEEP:
            oracle.forward(vals, meta, sc, li.L, li.R, li.X[:M])
            nbytes += algorithmic_bytes(SPEC.K, SPEC.N, SPEC.r, M)
            calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{calls} oracle forward calls (M in {list(M_SWEEP)}, one layer, fp64 numpy) in {el:.1f} s"}


def run_reference(args):
    # The oracle runs on rank 0's host cores only; the other ranks exit at once
    # (no process group: the reference arm has no collective step).
    if int(os.environ.get("RANK", "0")) != 0:
        return
    cb = cpu_baseline(budget_s=max(2.0, min(20.0, 2.0 * (args.steps + args.warmup))))
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD, "K": SPEC.K, "N": SPEC.N, "r": SPEC.r, "M": list(M_SWEEP)},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_slim(args):
    import torch
    ws, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from sparse_int4_linear_b200 import slim

    K, N, r = SPEC.K, SPEC.N, SPEC.r
    li = make_layer(SPEC, max(M_SWEEP))

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    base = slim.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
    layers = [base]
    for _ in range(args.layers - 1):
        lay = slim.PackedLayer(K, N, r, dev)
        lay._base.copy_(base._base)
        layers.append(lay)
    torch.cuda.synchronize()
    Xs = {M: to_dev(li.X[:M]) for M in M_SWEEP}
    Ys = {M: torch.empty(M, N, dtype=torch.bfloat16, device=dev) for M in M_SWEEP}
    wsp = slim.workspace(base, max(M_SWEEP), dev)

    # Parity of this exact configuration before timing (sampled output rows).
    parity = None
    if rank == 0:
        import oracle
        rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(1).choice(N, 62, replace=False)]))
        vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(li.W[rows]))
        worst = (0.0, 0.0)
        for M in M_SWEEP:
            Y = slim.linear(layers[-1], Xs[M], Ys[M], wsp)
            ref = oracle.forward(vals, meta, sc, li.L, np.ascontiguousarray(li.R[:, rows]), li.X[:M])
            e = oracle.errors(Y.float().cpu().numpy()[:, rows], ref)
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        parity = {"rel_fro": worst[0], "max_abs_rel": worst[1], "rows_checked": int(len(rows)),
                  "pass": bool(worst[0] <= oracle.REL_FRO_TOL and worst[1] <= oracle.MAX_ABS_TOL)}
        if not parity["pass"]:
            raise SystemExit(f"parity check failed before timing: {parity}")

    stream = torch.cuda.Stream(device=dev)

    def step(ms=M_SWEEP):
        for M in ms:
            for lay in layers:
                slim.linear(lay, Xs[M], Ys[M], wsp, stream=stream)

    # warm up the launch path (sets kernel attributes) before capture
    with torch.cuda.stream(stream):
        step()
    stream.synchronize()

    def capture(ms):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            step(ms)
        return g

    graph = capture(M_SWEEP)
    bytes_step = sum(algorithmic_bytes(K, N, r, M) for M in M_SWEEP) * len(layers)
    flops_step = sum(kept_flops(K, N, r, M) for M in M_SWEEP) * len(layers)
    calls_step = len(M_SWEEP) * len(layers)
    launches_step = sum(base.launches(M) for M in M_SWEEP) * len(layers)

    # CUDAGraph.replay() launches on torch's current stream: make it `stream`
    # so the events below bracket the replays.
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks, torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    el_ms = ev0.elapsed_time(ev1)
    el_max = max_over_ranks(el_ms, ws)
    value = bytes_step * args.steps * ws / (el_max / 1e3) / 1e9
    hbm_peak, tc_peak, peak_kind = load_peaks()

    # End to end through the host-buffer entry point (pinned X in, Y out): every
    # call enqueues its copies and forward; the step ends when its results are
    # on the host (one stream synchronisation per step).
    xh = {M: torch.from_numpy(li.X[:M].view(np.int16)).view(torch.bfloat16).pin_memory() for M in M_SWEEP}
    yh = {M: torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for M in M_SWEEP}
    hws = torch.zeros(base.host_workspace_bytes(max(M_SWEEP)), dtype=torch.uint8, device=dev)
    e2e_steps = max(1, min(args.steps, 20))

    def e2e_step():
        for M in M_SWEEP:
            for lay in layers:
                slim.linear_host(lay, xh[M], yh[M], hws, stream=stream, wait=False)
        stream.synchronize()

    e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws)
    e2e_value = bytes_step * e2e_steps * ws / (e2e_ms / 1e3) / 1e9
    h2d = sum(M * K * 2 for M in M_SWEEP) * len(layers)
    d2h = sum(M * N * 2 for M in M_SWEEP) * len(layers)

    per_m, cublas = {}, {}
    cb = None
    if rank == 0:
        # Per-M breakdown (separate graphs, after the timed region).
        for M in M_SWEEP:
            g = capture((M,))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = max(5, args.steps // 2)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    g.replay()
                a.record(stream)
                for _ in range(reps):
                    g.replay()
                b.record(stream)
            torch.cuda.synchronize()
            us = a.elapsed_time(b) * 1e3 / (reps * len(layers))
            gbs = algorithmic_bytes(K, N, r, M) / (us * 1e-6) / 1e9
            per_m[str(M)] = {"us_per_call": round(us, 3), "GB/s": round(gbs, 1),
                             "frac_hbm": round(gbs / hbm_peak, 4)}
        # Dense bf16 cuBLAS on the same shape (context; rotating weights).
        Wd = to_dev(li.W)
        Ld, Rd = to_dev(li.L), to_dev(li.R)
        n_copies = max(8, int(4 * 126e6 // (K * N * 2)) + 1)
        Wc = [Wd.clone() for _ in range(n_copies)]
        for M in M_SWEEP:
            for with_ad in (False, True):
                def dense(M=M, with_ad=with_ad):
                    for Wi in Wc:
                        y = torch.matmul(Xs[M], Wi.t())
                        if with_ad:
                            y = y + torch.matmul(torch.matmul(Xs[M], Ld), Rd)
                with torch.cuda.stream(stream):
                    dense()
                stream.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                reps = 10
                with torch.cuda.stream(stream):
                    a.record(stream)
                    for _ in range(reps):
                        dense()
                    b.record(stream)
                torch.cuda.synchronize()
                us = a.elapsed_time(b) * 1e3 / (reps * n_copies)
                key = f"M{M}" + ("+adapter" if with_ad else "")
                cublas[key] = {"us_per_call": round(us, 3)}
        for M in M_SWEEP:
            cublas[f"M{M}+adapter"]["slim_speedup"] = round(cublas[f"M{M}+adapter"]["us_per_call"]
                                                            / per_m[str(M)]["us_per_call"], 3)
        if args.gpus == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline()

    # Roofline of the dominant kernel (the single-launch decode kernel, one
    # launch per M = 1 call): algorithmic bytes of a call over its time in the
    # M = 1 graph replays (CUDA events on the replay stream).
    achieved = per_m["1"]["GB/s"] if per_m else None
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, torch CPU RNG)",
        "config": {"workload": WORKLOAD, "K": K, "N": N, "r": r, "group": 128, "M": list(M_SWEEP),
                   "layers_per_step": len(layers), "calls_per_step": calls_step,
                   "l2": f"inputs larger than L2: {len(layers)} packed copies, "
                         f"{len(layers) * algorithmic_bytes(K, N, r, 0) / 1e6:.0f} MB read per M pass",
                   "cuda_graph": True, "parallelism": f"replicas x{ws}"},
        "roofline": {"kernel": "k_stream (single-launch decode), M = 1 calls", "bound": "hbm",
                     "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4) if achieved else None, "peak_kind": peak_kind,
                     "traffic": TRAFFIC_M1_LAUNCH if base.launches(1) == 1 else None,
                     "algorithmic_bytes_per_launch": algorithmic_bytes(K, N, r, 1),
                     "timed": "graph replays of the 60 M = 1 calls, CUDA events on the replay stream"},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "api": "slim_linear_host_async per call (pinned X -> device, forward, Y -> pinned host), "
                       "one stream synchronisation per step"},
        "gpu_launches": launches_step * args.steps,
        "clocks": clocks.summary(),
        "parity": parity,
        "per_m": per_m,
        "tflops": round(flops_step * args.steps * ws / (el_max / 1e3) / 1e12, 3),
        "cublas_dense_bf16": cublas,
        "cpu_baseline": cb,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- prefill workload
PREFILL_SPECS = CONFIGS[3][0]      # 7B up_proj 4096 -> 11008 and down_proj 11008 -> 4096, r = 128
PREFILL_M = CONFIGS[3][1][0]       # 2048 tokens
PREFILL_METRIC = METRIC
PREFILL_WORKLOAD = "LLaMA-2-7B MLP up (4096->11008) + down (11008->4096), prefill M=2048, g=128 int4 + 2:4, r=128"


def run_prefill(args):
    """One step = the up and the down projection of one M = 2048 batch (TFLOP/s of kept + adapter FLOPs)."""
    import torch
    ws_n, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from sparse_int4_linear_b200 import slim

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    M = PREFILL_M
    layers, Xs, Ys, wss, flops = [], [], [], [], 0
    parity = []
    for spec in PREFILL_SPECS:
        li = make_layer(spec, M)
        lay = slim.pack(to_dev(li.W), to_dev(li.L), to_dev(li.R))
        X = to_dev(li.X)
        Y = torch.empty(M, spec.N, dtype=torch.bfloat16, device=dev)
        wsp = slim.workspace(lay, M, dev)
        if rank == 0:
            import oracle
            rows = np.unique(np.concatenate([[0, spec.N - 1], np.random.default_rng(2).choice(spec.N, 30, replace=False)]))
            vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(li.W[rows]))
            slim.linear(lay, X, Y, wsp)
            ref = oracle.forward(vals, meta, sc, li.L, np.ascontiguousarray(li.R[:, rows]), li.X)
            e = oracle.errors(Y.float().cpu().numpy()[:, rows], ref)
            parity.append({"layer": spec.name, "rel_fro": e[0], "max_abs_rel": e[1]})
        layers.append(lay); Xs.append(X); Ys.append(Y); wss.append(wsp)
        flops += kept_flops(spec.K, spec.N, spec.r, M)
    stream = torch.cuda.Stream(device=dev)

    def step():
        for lay, X, Y, w in zip(layers, Xs, Ys, wss):
            slim.linear(lay, X, Y, w, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    barrier(ws_n)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks, torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws_n)
    el = max_over_ranks(ev0.elapsed_time(ev1), ws_n)
    value = flops * args.steps * ws_n / (el / 1e3) / 1e12
    _, tc_peak, peak_kind = load_peaks()
    achieved = flops / (el / 1e3 / args.steps) / 1e12
    line = {"metric": PREFILL_METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, torch CPU RNG)",
            "config": {"workload": PREFILL_WORKLOAD, "M": M, "layers": [s.name for s in PREFILL_SPECS],
                       "l2": "2 layers + X per step; X and weights stay L2-resident across calls (compute-bound)"},
            "roofline": {"kernel": "slim_linear prefill (all kernels of the call)", "bound": "tensor",
                         "achieved": round(achieved, 1), "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": round(achieved / tc_peak, 4), "peak_kind": peak_kind + " dense bf16 (burst)",
                         "traffic": None},
            "gpu_launches": sum(lay.launches(M) for lay in layers) * args.steps,
            "clocks": clocks.summary(), "parity": parity}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- decoder-block workload
BLOCK_SPECS, BLOCK_M = CONFIGS[4]   # LLaMA-2-7B block: q, k, v, o, gate, up, down; r = 128
BLOCK_WORKLOAD = ("LLaMA-2-7B decoder block (q, k, v, o 4096x4096; gate, up 4096->11008; down 11008->4096), "
                  "g=128 int4 + 2:4, r=128, M in {1, 16, 256, 1024, 4096}")


def run_block(args):
    """One step = the 7 linears of a block at one M, as one CUDA graph over
    rotating copies (cold L2).  Timed twice: 7 separate layers, and fused
    (q, k, v as one grouped layer; gate, up as one; o; down: 4 calls)."""
    import torch
    ws_n, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from sparse_int4_linear_b200 import slim

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    Mmax = max(BLOCK_M)
    lis = {s.name.split(".")[1]: make_layer(s, Mmax) for s in BLOCK_SPECS}
    W = {k: to_dev(v.W) for k, v in lis.items()}
    Ld = {k: to_dev(v.L) for k, v in lis.items()}
    Rd = {k: to_dev(v.R) for k, v in lis.items()}
    X4 = to_dev(lis["q"].X)          # [Mmax][4096]: the input of q, k, v, o, gate, up
    X11 = to_dev(lis["down"].X)      # [Mmax][11008]: the input of down
    sep0 = {k: slim.pack(W[k], Ld[k], Rd[k]) for k in lis}
    fused0 = {"qkv": slim.pack_grouped([W["q"], W["k"], W["v"]], [Ld["q"], Ld["k"], Ld["v"]],
                                       [Rd["q"], Rd["k"], Rd["v"]]),
              "o": sep0["o"],
              "gateup": slim.pack_grouped([W["gate"], W["up"]], [Ld["gate"], Ld["up"]], [Rd["gate"], Rd["up"]]),
              "down": sep0["down"]}
    del W, Ld, Rd
    block_bytes0 = sum(algorithmic_bytes(s.K, s.N, s.r, 0) for s in BLOCK_SPECS)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = int(np.ceil(4 * l2 / block_bytes0)) + 1

    def clone(lay):
        c = slim.PackedLayer(lay.K, lay.N_list, lay.r, dev)
        c._base.copy_(lay._base)
        return c

    seps = [sep0] + [{k: clone(v) for k, v in sep0.items()} for _ in range(copies - 1)]
    fuseds = [fused0] + [{"qkv": clone(fused0["qkv"]), "o": c["o"], "gateup": clone(fused0["gateup"]),
                          "down": c["down"]} for c in seps[1:]]
    torch.cuda.synchronize()

    # Parity of the fused block against the oracle (sampled rows, M = 16).
    parity = None
    if rank == 0:
        import oracle
        rows = np.array([0, 1, 777, 4095])
        worst = (0.0, 0.0)
        Yq = slim.linear(fused0["qkv"], X4[:16])
        Yg = slim.linear(fused0["gateup"], X4[:16])
        Yd = slim.linear(fused0["down"], X11[:16])
        for name, Y, off, li, Xb in (("q", Yq, 0, lis["q"], lis["q"].X), ("v", Yq, 8192, lis["v"], lis["q"].X),
                                     ("up", Yg, 11008, lis["up"], lis["q"].X), ("down", Yd, 0, lis["down"], lis["down"].X)):
            vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(li.W[rows]))
            ref = oracle.forward(vals, meta, sc, li.L, np.ascontiguousarray(li.R[:, rows]), Xb[:16])
            e = oracle.errors(Y.float().cpu().numpy()[:, off + rows], ref)
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        parity = {"rel_fro": worst[0], "max_abs_rel": worst[1], "pass": bool(worst[0] <= oracle.REL_FRO_TOL and
                                                                             worst[1] <= oracle.MAX_ABS_TOL)}
        if not parity["pass"]:
            raise SystemExit(f"parity check failed before timing: {parity}")

    stream = torch.cuda.Stream(device=dev)
    hbm_peak, tc_peak, peak_kind = load_peaks()
    per_m = {}
    dec_bytes = dec_us = 0.0
    launches = 0
    with ClockSampler(local) as clocks:
        for M in BLOCK_M:
            Y4 = torch.empty(M, 4096, dtype=torch.bfloat16, device=dev)
            Y11 = torch.empty(M, 11008, dtype=torch.bfloat16, device=dev)
            Yqkv = torch.empty(M, 3 * 4096, dtype=torch.bfloat16, device=dev)
            Ygu = torch.empty(M, 2 * 11008, dtype=torch.bfloat16, device=dev)
            need = max([l.workspace_bytes(M) for c in seps for l in c.values()] +
                       [l.workspace_bytes(M) for c in fuseds for l in c.values()])
            wsp = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
            xa, xd = X4[:M], X11[:M]

            def run_sep():
                for c in seps:
                    for k in ("q", "k", "v", "o"):
                        slim.linear(c[k], xa, Y4, wsp, stream=stream)
                    slim.linear(c["gate"], xa, Y11, wsp, stream=stream)
                    slim.linear(c["up"], xa, Y11, wsp, stream=stream)
                    slim.linear(c["down"], xd, Y4, wsp, stream=stream)

            def run_fused():
                for c in fuseds:
                    slim.linear(c["qkv"], xa, Yqkv, wsp, stream=stream)
                    slim.linear(c["o"], xa, Y4, wsp, stream=stream)
                    slim.linear(c["gateup"], xa, Ygu, wsp, stream=stream)
                    slim.linear(c["down"], xd, Y4, wsp, stream=stream)

            res = {}
            for tag, fn in (("separate", run_sep), ("fused", run_fused)):
                with torch.cuda.stream(stream):
                    fn()
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                    fn()
                reps = 10 if M <= 16 else 5
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    for _ in range(max(3, args.warmup)):
                        g.replay()
                    a.record(stream)
                    for _ in range(reps):
                        g.replay()
                    b.record(stream)
                torch.cuda.synchronize()
                res[tag] = a.elapsed_time(b) * 1e3 / (reps * copies)   # us per block
                del g
            bytes_blk = sum(algorithmic_bytes(s.K, s.N, s.r, M) for s in BLOCK_SPECS)
            flops_blk = sum(kept_flops(s.K, s.N, s.r, M) for s in BLOCK_SPECS)
            entry = {"us_per_block_separate": round(res["separate"], 2), "us_per_block_fused": round(res["fused"], 2),
                     "fused_speedup": round(res["separate"] / res["fused"], 3),
                     "launches_separate": sum(l.launches(M) for l in sep0.values()),
                     "launches_fused": sum(l.launches(M) for l in fused0.values())}
            if M <= 16:
                gbs = bytes_blk / (res["fused"] * 1e-6) / 1e9
                entry.update({"GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4)})
                dec_bytes += bytes_blk
                dec_us += res["fused"]
            else:
                tf = flops_blk / (res["fused"] * 1e-6) / 1e12
                entry.update({"TFLOP/s": round(tf, 1), "frac_tensor": round(tf / tc_peak, 4)})
            per_m[str(M)] = entry
            launches += entry["launches_fused"]
    value = dec_bytes / (dec_us * 1e-6) / 1e9
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws_n, "steps": 1,
            "warmup": max(3, args.warmup), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded, torch CPU RNG)",
            "config": {"workload": BLOCK_WORKLOAD, "copies": copies,
                       "l2": f"{copies} rotating copies of the block ({copies * block_bytes0 / 1e6:.0f} MB), cold L2",
                       "value_is": "fused block, M = 1 and 16: algorithmic bytes / time", "cuda_graph": True},
            "roofline": {"kernel": "fused block (4 calls), M = 1 and 16", "bound": "hbm", "achieved": round(value, 1),
                         "peak": hbm_peak, "unit": "GB/s", "frac": round(value / hbm_peak, 4),
                         "peak_kind": peak_kind, "traffic": None},
            "gpu_launches": launches, "clocks": clocks.summary(), "parity": parity, "per_m": per_m}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["slim", "reference"], default="slim")
    ap.add_argument("--layers", type=int, default=60, help="packed copies of the layer per step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["decode", "prefill", "block"], default="decode",
                    help="decode: 7B q_proj M in {1,4,16} (the default line); prefill: 7B MLP at M = 2048; "
                         "block: the 7 linears of a 7B decoder block, separate and fused, M in {1..4096}")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefill":
        run_prefill(args)
    elif args.workload == "block":
        run_block(args)
    else:
        run_slim(args)


if __name__ == "__main__":
    main()
