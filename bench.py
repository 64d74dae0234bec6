#!/usr/bin/env python3
"""Benchmark of the compressed linear layer on one B200.

Headline workload: the LLaMA-2-70B-shaped linears (q 8192x8192; k, v
8192->1024; gate, up 8192->28672; down 28672->8192), int4 2:4 weights with
group-128 fp16 scales and an r = 256 bf16 adapter, synthetic seeded inputs.

* value (GB/s): one step = the six layers at decode batches M = 1 and M = 16,
  pushed through enough independently packed copies of the six-layer set
  (ceil(4 * L2 / set bytes) + 1) that every call reads its weights from HBM,
  captured once as a CUDA graph per M and replayed.  The metric is
  algorithmic bytes per second: packed values + metadata + scales + L + R + X
  + Y of every call (the decode regime is memory-bound; thesis §2.5.2).
* prefill (TFLOP/s): the six layers at M = 512 and M = 4096, kept (2:4) MACs
  plus the adapter's, per second (compute-bound; thesis §2.5.1), against the
  measured dense bf16 peak (the sparse tensor cores process kept MACs at the
  dense MAC rate).
* per-config fields: the 7B q_proj decode sweep (K = N = 4096, r = 128,
  M in {1, 4, 16}) and the 7B MLP pair at M = 2048.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl slim|reference]
                    [--workload headline|block]

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas, no collective on the data path); the whole-job value
is the sum of the ranks' bytes over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_int4_linear_b200.workload import CONFIGS, make_layer  # noqa: E402

METRIC = "2:4+INT4+low-rank linear: GB/s (M≤16), TFLOP/s (M≥256) vs B200 roofline"
HEAD_SPECS = CONFIGS[5][0]                 # 70B q, k, v, gate, up, down; r = 256
DECODE_M = (1, 16)
PREFILL_M = (512, 4096)
WORKLOAD = ("LLaMA-2-70B-shaped linears (q 8192x8192; k, v 8192->1024; gate, up 8192->28672; down 28672->8192), "
            "g=128 int4 + 2:4, adapter r=256 bf16; value: decode M in {1,16}; prefill: M in {512,4096}")
Q7_SPEC, Q7_M = CONFIGS[2][0][0], (1, 4, 16)        # 7B q_proj decode sweep
MLP7_SPECS, MLP7_M = CONFIGS[3][0], CONFIGS[3][1][0]  # 7B up + down, M = 2048
CPU_SAMPLE_SPEC = CONFIGS[5][0][1]                    # 70B k (8192 -> 1024): the smallest layer of the set


def algorithmic_bytes(K, N, r, M):
    """vals + meta + scales + L + R + X + Y (the T = X L scratch excluded)."""
    return N * K // 4 + N * K // 8 + N * (K // 128) * 2 + 2 * K * r + 2 * r * N + 2 * M * K + 2 * M * N


def algorithmic_bytes_q4(K, N, r, M):
    """As algorithmic_bytes, with L and R stored as 4-bit fragments plus fp16
    scales (one per 128 entries along each factor's reduction dimension)."""
    r16 = -(-r // 16) * 16
    lq = r16 // 16 * (K // 128) * 1056
    rq = -(-N // 16) * (r16 // 16 * 128 + -(-r // 128) * 32)
    return N * K // 4 + N * K // 8 + N * (K // 128) * 2 + lq + rq + 2 * M * K + 2 * M * N


def kept_flops(K, N, r, M):
    """2 per kept (2:4) MAC of the main product plus the adapter's X L and T R."""
    return 2 * M * N * (K // 2) + 2 * M * r * (K + N)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)) or None, \
            "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- ncu traffic
def committed_traffic(kernel_tag: str):
    """DRAM bytes per launch of a kernel from the committed ncu summary under
    profiles/, used only while the kernel's sources are unchanged since that
    capture (the summary records their sha256); otherwise None."""
    prof = os.path.join(ROOT, "profiles")
    if not os.path.isdir(prof):
        return None
    for fn in sorted(os.listdir(prof)):
        if not fn.endswith(".md"):
            continue
        txt = open(os.path.join(prof, fn)).read()
        m = re.search(r"traffic-record: kernel=(\S+) workload=(\S+) bytes_per_launch=(\d+) sources=(\S+) "
                      r"sha256=([0-9a-f]{64})", txt)
        if not m or m.group(1) != kernel_tag:
            continue
        files = m.group(4).split(",")
        h = hashlib.sha256()
        for f in files:
            path = os.path.join(ROOT, f)
            if not os.path.exists(path):
                return None
            h.update(open(path, "rb").read())
        if h.hexdigest() != m.group(5):
            return None
        return {"bytes_per_launch": int(m.group(3)), "workload": m.group(2), "summary": f"profiles/{fn}"}
    return None


def decode_roofline(specs, launches1, per_layer, per_m, hbm_peak, peak_kind, traffic, copies):
    """Roofline object of the dominant decode kernel, k_stream, at M = 1: the
    layers whose one-token call is a single k_stream launch, their algorithmic
    bytes over the sum of their per-call times (per-layer graphs of rotating
    copies, CUDA events).  Without such layers: the whole M = 1 set."""
    ks = [s for s in specs if launches1[s.name] == 1]
    if ks:
        kb = sum(algorithmic_bytes(s.K, s.N, s.r, 1) for s in ks)
        kus = sum(per_layer[s.name]["1"]["us"] for s in ks)
        ach = round(kb / (kus * 1e-6) / 1e9, 1)
        kernel = ("k_stream (single-launch decode, one launch per call) at M = 1 on "
                  + ", ".join(s.name for s in ks))
        timed = (f"per-layer CUDA graphs of rotating copies of each of these layers (cold L2), CUDA events on the "
                 f"replay stream; achieved = their algorithmic bytes ({kb} B, one launch each) / the sum of their "
                 f"per-call times ({kus:.2f} us); the whole M = 1 set is per_m['1']")
    else:
        ach = per_m["1"]["GB/s"]
        kernel = "slim_linear decode calls at M = 1"
        timed = (f"median of 100 replays of the M = 1 graph ({copies} x {len(specs)} calls), CUDA events on the "
                 "replay stream; achieved = algorithmic bytes of the calls / time")
    return {"kernel": kernel, "bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
            "frac": round(ach / hbm_peak, 4), "peak_kind": f"{peak_kind} HBM copy bandwidth",
            "traffic": traffic["bytes_per_launch"] if traffic and ks else None,
            "traffic_source": traffic if ks else None,
            "algorithmic_bytes_per_launch": {s.name: algorithmic_bytes(s.K, s.N, s.r, 1) for s in specs},
            "timed": timed}


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
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(budget_s: float = 10.0, threads: int | None = None):
    """The oracle forward as it stands, timed on the host cores on a bounded
    sample of the headline workload: repeated decode calls (M = 1 and 16) of
    its smallest layer, the 70B k projection (8192 -> 1024, r = 256), until
    ~budget_s.  threads=1 pins the BLAS pool to one thread."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    spec = CPU_SAMPLE_SPEC
    li = make_layer(spec, max(DECODE_M))
    vals, meta, sc = oracle.pack_layer(li.W)

    def run():
        nbytes, calls = 0, 0
        t0 = time.perf_counter()
        while True:
            for M in DECODE_M:
                oracle.forward(vals, meta, sc, li.L, li.R, li.X[:M])
                nbytes += algorithmic_bytes(spec.K, spec.N, spec.r, M)
                calls += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                return nbytes, calls, el

    if threads:
        with threadpool_limits(limits=threads):
            nbytes, calls, el = run()
        cores = threads
    else:
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
        nbytes, calls, el = run()
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": int(cores), "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": f"{calls} oracle forward calls (70B k 8192->1024, r=256, M in {list(DECODE_M)}; "
                      f"fp64 numpy, pack excluded) in {el:.1f} s"}


def run_reference(args):
    # The oracle runs on rank 0's host cores only; the other ranks exit at once
    # (no process group: the reference arm has no collective step).
    if int(os.environ.get("RANK", "0")) != 0:
        return
    cb = cpu_baseline(budget_s=max(2.0, min(20.0, 2.0 * (args.steps + args.warmup))))
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD, "value_is": "decode M in {1,16}: algorithmic bytes / time",
                       "sample_layer": CPU_SAMPLE_SPEC.name},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU helpers
def _to_dev(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


def _clone_layer(slim, lay, dev):
    c = slim.PackedLayer(lay.K, lay.N_list if len(lay.N_list) > 1 else lay.N, lay.r, dev)
    c.set_adapter_bits(lay.adapter_bits)
    c._base.copy_(lay._base)
    return c


def _capture(torch, fn, stream):
    torch.cuda.synchronize()          # buffers zero-filled on other streams are ready
    with torch.cuda.stream(stream):   # warm the launch path (kernel attributes) before capture
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        fn()
    return g


def _time_replays(torch, graphs, stream, reps, warmup=3):
    """Per-replay times (ms) of one replay of every graph in `graphs`,
    CUDA events on the replay stream."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            for g in graphs:
                g.replay()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    with torch.cuda.stream(stream):
        evs[0].record(stream)
        for i in range(reps):
            for g in graphs:
                g.replay()
            evs[i + 1].record(stream)
    torch.cuda.synchronize()
    return [evs[i].elapsed_time(evs[i + 1]) for i in range(reps)]


def _pcts(x):
    a = np.asarray(x, dtype=np.float64)
    return float(np.median(a)), float(np.percentile(a, 10)), float(np.percentile(a, 90))


def _parity(slim, oracle, torch, lay, li, X_dev, M, dev, n_rows=24, seed=1):
    """Sampled output rows of one call against the fp64 oracle (its 4-bit
    adapter forward for a layer packed with 4-bit adapters)."""
    N = lay.N
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(seed).choice(N, min(N, n_rows),
                                                                                    replace=False)]))
    Y = slim.linear(lay, X_dev[:M])
    vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(li.W[rows]))
    fwd = oracle.forward_quantized_adapters if lay.adapter_bits == 4 else oracle.forward
    ref = fwd(vals, meta, sc, li.L, np.ascontiguousarray(li.R[:, rows]), li.X[:M])
    return oracle.errors(Y.float().cpu().numpy()[:, rows], ref)


# ---------------------------------------------------------------- headline
def run_headline(args):
    import torch
    ws, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from sparse_int4_linear_b200 import slim
    import oracle

    hbm_peak, tc_peak, tc_sust, peak_kind = load_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    names = [s.name for s in HEAD_SPECS]
    Mmax = max(PREFILL_M)

    # ---- pack the six layers, parity of sampled rows before timing
    base, Xd, parity = {}, {}, []
    for spec in HEAD_SPECS:
        li = make_layer(spec, Mmax)
        base[spec.name] = slim.pack(_to_dev(li.W, dev), _to_dev(li.L, dev), _to_dev(li.R, dev))
        Xd[spec.name] = _to_dev(li.X, dev)
        if rank == 0:
            for M in (1, 16, 512):
                e = _parity(slim, oracle, torch, base[spec.name], li, Xd[spec.name], M, dev, seed=spec.seed)
                parity.append({"layer": spec.name, "M": M, "rel_fro": e[0], "max_abs_rel": e[1]})
        del li
    if rank == 0:
        worst = (max(p["rel_fro"] for p in parity), max(p["max_abs_rel"] for p in parity))
        ok = worst[0] <= oracle.REL_FRO_TOL and worst[1] <= oracle.MAX_ABS_TOL
        parity = {"rel_fro": worst[0], "max_abs_rel": worst[1], "pass": bool(ok),
                  "checked": "26 sampled output rows of every layer at M = 1, 16 and 512 vs the fp64 oracle"}
        if not ok:
            raise SystemExit(f"parity check failed before timing: {parity}")

    # ---- decode: rotating copies of the six-layer set (cold L2)
    set_bytes = sum(algorithmic_bytes(s.K, s.N, s.r, 0) for s in HEAD_SPECS)
    copies = int(np.ceil(4 * l2 / set_bytes)) + 1
    sets = [base] + [{n: _clone_layer(slim, base[n], dev) for n in names} for _ in range(copies - 1)]
    Ydec = {(n, M): torch.empty(M, base[n].N, dtype=torch.bfloat16, device=dev) for n in names for M in DECODE_M}
    wsp = torch.zeros(max(max(base[n].workspace_bytes(max(DECODE_M)) for n in names), 16), dtype=torch.uint8,
                      device=dev)

    def dec_calls(M):
        def fn():
            for s in sets:
                for n in names:
                    slim.linear(s[n], Xd[n][:M], Ydec[(n, M)], wsp, stream=stream)
        return fn

    gdec = {M: _capture(torch, dec_calls(M), stream) for M in DECODE_M}
    bytes_m = {M: copies * sum(algorithmic_bytes(s.K, s.N, s.r, M) for s in HEAD_SPECS) for M in DECODE_M}
    bytes_step = sum(bytes_m.values())
    launches_step = copies * sum(base[n].launches(M) for n in names for M in DECODE_M)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for M in DECODE_M:
                gdec[M].replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks, torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            for M in DECODE_M:
                gdec[M].replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    el_ms = max_over_ranks(ev0.elapsed_time(ev1), ws)
    value = bytes_step * args.steps * ws / (el_ms / 1e3) / 1e9

    # ---- end to end through the host-buffer entry point
    xh = {(n, M): Xd[n][:M].cpu().pin_memory() for n in names for M in DECODE_M}
    yh = {(n, M): torch.empty(M, base[n].N, dtype=torch.bfloat16).pin_memory() for n in names for M in DECODE_M}
    hws = torch.zeros(max(base[n].host_workspace_bytes(max(DECODE_M)) for n in names), dtype=torch.uint8,
                      device=dev)
    e2e_steps = max(1, min(args.steps, 20))
    torch.cuda.synchronize()

    def e2e_calls():
        for M in DECODE_M:
            for s in sets:
                for n in names:
                    slim.linear_host(s[n], xh[(n, M)], yh[(n, M)], hws, stream=stream, wait=False)

    def time_e2e(step):
        step()
        torch.cuda.synchronize()
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), ws)

    # (a) The host-buffer entry point, call by call (each call copies its X in
    # and its Y out on the stream).
    def e2e_step_calls():
        e2e_calls()
        stream.synchronize()

    e2e_ms_calls = time_e2e(e2e_step_calls)
    # (b) The step's inputs staged in one pinned buffer: one copy of all of
    # them to the device, slim_linear per call on device views, one copy of
    # all outputs back; captured once as a CUDA graph (the copies are nodes of
    # the graph, so they run every replay).  Every call has its own X and Y
    # bytes, as in (a).
    order = [(s_i, n, M) for M in DECODE_M for s_i in range(len(sets)) for n in names]
    x_off, y_off, xo, yo = {}, {}, 0, 0
    for key in order:
        _, n, M = key
        x_off[key], y_off[key] = xo, yo
        xo += M * base[n].K
        yo += M * base[n].N
    xin = torch.empty(xo, dtype=torch.bfloat16).pin_memory()
    for (s_i, n, M), o in x_off.items():
        xin[o:o + M * base[n].K] = xh[(n, M)].reshape(-1)
    yout = torch.empty(yo, dtype=torch.bfloat16).pin_memory()
    xdev = torch.empty(xo, dtype=torch.bfloat16, device=dev)
    ydev = torch.empty(yo, dtype=torch.bfloat16, device=dev)

    def e2e_staged():
        xdev.copy_(xin, non_blocking=True)
        for (s_i, n, M) in order:
            xv = xdev[x_off[(s_i, n, M)]:x_off[(s_i, n, M)] + M * base[n].K].view(M, base[n].K)
            yv = ydev[y_off[(s_i, n, M)]:y_off[(s_i, n, M)] + M * base[n].N].view(M, base[n].N)
            slim.linear(sets[s_i][n], xv, yv, wsp, stream=stream)
        yout.copy_(ydev, non_blocking=True)

    g_e2e = _capture(torch, e2e_staged, stream)

    def e2e_step_graph():
        with torch.cuda.stream(stream):
            g_e2e.replay()
        stream.synchronize()

    e2e_ms = time_e2e(e2e_step_graph)
    del g_e2e
    e2e_value = bytes_step * e2e_steps * ws / (e2e_ms / 1e3) / 1e9
    e2e_value_calls = bytes_step * e2e_steps * ws / (e2e_ms_calls / 1e3) / 1e9
    h2d = copies * sum(M * s.K * 2 for s in HEAD_SPECS for M in DECODE_M)
    d2h = copies * sum(M * s.N * 2 for s in HEAD_SPECS for M in DECODE_M)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, torch CPU RNG)",
        "config": {"workload": WORKLOAD, "layers": names, "r": 256, "group": 128, "M_decode": list(DECODE_M),
                   "M_prefill": list(PREFILL_M), "copies": copies,
                   "l2": f"inputs larger than L2: {copies} packed copies of the six-layer set, "
                         f"{copies * set_bytes / 1e6:.0f} MB of weights read per M pass (L2 {l2 / 1e6:.0f} MB)",
                   "value_is": "decode M in {1,16}: algorithmic bytes / time", "cuda_graph": True,
                   "parallelism": f"replicas x{ws}"},
        "gpu_launches": launches_step * args.steps,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "api": "the step's inputs in one pinned host buffer: one copy to the device, "
                                          "slim_linear per call on device views, one copy of all outputs back "
                                          "to pinned host memory, captured as one CUDA graph (copies included); "
                                          "one stream synchronisation per step",
                "value_host_entry_point_per_call": round(e2e_value_calls, 2),
                "host_entry_point": "slim_linear_host_async per call (its own X in and Y out), issued from "
                                    "Python, one stream synchronisation per step"},
        "clocks": clocks.summary(),
        "parity": parity,
    }

    if rank == 0:
        # ---- statistics and per-M / per-layer breakdown (after the timed region)
        stats = []
        for _ in range(3):
            t = _time_replays(torch, [gdec[M] for M in DECODE_M], stream, reps=max(100, args.steps))
            stats.append([bytes_step / (x / 1e3) / 1e9 for x in t])
        allv = [v for s in stats for v in s]
        med, p10, p90 = _pcts(allv)
        line["value_stats"] = {"median": round(med, 1), "p10": round(p10, 1), "p90": round(p90, 1),
                               "repeat_medians": [round(float(np.median(s)), 1) for s in stats],
                               "iterations": len(allv), "unit": "GB/s"}
        per_m = {}
        for M in DECODE_M:
            t = _time_replays(torch, [gdec[M]], stream, reps=100)
            med, p10, p90 = _pcts(t)
            calls = copies * len(names)
            gbs = bytes_m[M] / (med / 1e3) / 1e9
            per_m[str(M)] = {"us_per_set": round(med * 1e3 / copies, 2), "GB/s": round(gbs, 1),
                             "frac_hbm": round(gbs / hbm_peak, 4),
                             "p10_p90_GB/s": [round(bytes_m[M] / (p90 / 1e3) / 1e9, 1),
                                              round(bytes_m[M] / (p10 / 1e3) / 1e9, 1)],
                             "launches_per_call": [base[n].launches(M) for n in names], "calls": calls}
        line["per_m"] = per_m
        # per layer: rotating copies of that layer alone, enough to exceed 4x L2
        per_layer = {}
        for spec in HEAD_SPECS:
            n = spec.name
            lb = algorithmic_bytes(spec.K, spec.N, spec.r, 0)
            nc = min(int(np.ceil(4 * l2 / lb)) + 1, 80)
            cl = [base[n]] + [_clone_layer(slim, base[n], dev) for _ in range(nc - 1)]
            ent = {}
            for M in DECODE_M:
                def fn(M=M, cl=cl, n=n):
                    for c in cl:
                        slim.linear(c, Xd[n][:M], Ydec[(n, M)], wsp, stream=stream)
                g = _capture(torch, fn, stream)
                us = float(np.median(_time_replays(torch, [g], stream, reps=30))) * 1e3 / nc
                gbs = algorithmic_bytes(spec.K, spec.N, spec.r, M) / (us * 1e-6) / 1e9
                ent[str(M)] = {"us": round(us, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4)}
                del g
            per_layer[n] = ent
            del cl
            torch.cuda.empty_cache()
        line["per_layer_decode"] = per_layer

        # ---- roofline of the dominant kernel: the single-launch decode kernel at M = 1
        line["roofline"] = decode_roofline(HEAD_SPECS, {n: base[n].launches(1) for n in names}, per_layer, per_m,
                                           hbm_peak, peak_kind, committed_traffic("k_stream"), copies)

        # ---- the same decode set with 4-bit adapters (Quantized SLiM)
        del sets, gdec
        torch.cuda.empty_cache()
        line["adapter_int4"] = run_adapter_int4(torch, slim, oracle, dev, stream, l2, hbm_peak, Xd, per_m)

        # ---- prefill regime
        torch.cuda.empty_cache()
        pre = {}
        pws = torch.zeros(max(base[n].workspace_bytes(Mmax) for n in names), dtype=torch.uint8, device=dev)
        for M in PREFILL_M:
            Yp = {n: torch.empty(M, base[n].N, dtype=torch.bfloat16, device=dev) for n in names}

            def fn(M=M, Yp=Yp):
                for n in names:
                    slim.linear(base[n], Xd[n][:M], Yp[n], pws, stream=stream)
            g = _capture(torch, fn, stream)
            t = _time_replays(torch, [g], stream, reps=30)
            med, p10, p90 = _pcts(t)
            fl = sum(kept_flops(s.K, s.N, s.r, M) for s in HEAD_SPECS)
            tf = fl / (med / 1e3) / 1e12
            ent = {"us_per_set": round(med * 1e3, 1), "TFLOP/s": round(tf, 1), "frac_tensor": round(tf / tc_peak, 4),
                   "p10_p90_TFLOP/s": [round(fl / (p90 / 1e3) / 1e12, 1), round(fl / (p10 / 1e3) / 1e12, 1)],
                   "launches": sum(base[n].launches(M) for n in names), "per_layer_us": {}}
            for n, s in zip(names, HEAD_SPECS):
                def fl1(n=n, M=M, Yp=Yp):
                    slim.linear(base[n], Xd[n][:M], Yp[n], pws, stream=stream)
                g1 = _capture(torch, fl1, stream)
                us = float(np.median(_time_replays(torch, [g1], stream, reps=20))) * 1e3
                ent["per_layer_us"][n] = {"us": round(us, 1),
                                          "TFLOP/s": round(kept_flops(s.K, s.N, s.r, M) / (us * 1e-6) / 1e12, 1)}
                del g1
            pre[str(M)] = ent
            del g, Yp
        big = pre[str(max(PREFILL_M))]
        line["prefill"] = {
            "unit": "TFLOP/s", "per_m": pre,
            "roofline": {"kernel": "slim_linear prefill calls (T = X L, weight-image pass, sparse tcgen05 MMA), "
                                   f"the six 70B layers at M = {max(PREFILL_M)}", "bound": "tensor",
                         "achieved": big["TFLOP/s"], "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": round(big["TFLOP/s"] / tc_peak, 4),
                         "frac_of_sustained": round(big["TFLOP/s"] / tc_sust, 4) if tc_sust else None,
                         "peak_kind": f"{peak_kind} dense bf16 (burst); kept MACs run at the dense MAC rate",
                         "traffic": None}}
        del pws
        torch.cuda.empty_cache()

        # ---- dense bf16 cuBLAS on the same shapes (context)
        line["cublas_dense_bf16"] = dense_baseline(torch, dev, stream, l2, per_m, pre)

        # ---- per-config fields
        line["per_config"] = {"7b_q_proj_decode": run_q7(torch, slim, dev, stream, hbm_peak),
                              "7b_mlp_prefill_m2048": run_mlp7(torch, slim, dev, stream, tc_peak)}

        if args.gpus == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(10.0)
            line["cpu_baseline_1thread"] = cpu_baseline(8.0, threads=1)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_adapter_int4(torch, slim, oracle, dev, stream, l2, hbm_peak, Xd, per_m_bf16):
    """Decode of the six 70B layers with L and R quantized to 4 bits (thesis
    §7.4.3, Quantized SLiM), timed like the headline (rotating copies, cold
    L2): GB/s of the 4-bit layout's algorithmic bytes, and the time per set
    against the bf16-adapter set."""
    names = [s.name for s in HEAD_SPECS]
    q4, worst = {}, [0.0, 0.0]
    for spec in HEAD_SPECS:
        li = make_layer(spec, max(PREFILL_M))   # the X the headline drew (Xd), outlier channels included
        q4[spec.name] = slim.pack(_to_dev(li.W, dev), _to_dev(li.L, dev), _to_dev(li.R, dev), adapter_bits=4)
        for M in DECODE_M:
            e = _parity(slim, oracle, torch, q4[spec.name], li, Xd[spec.name], M, dev, seed=spec.seed + 1)
            worst = [max(worst[0], e[0]), max(worst[1], e[1])]
        del li
    ok = worst[0] <= oracle.REL_FRO_TOL and worst[1] <= oracle.MAX_ABS_TOL
    if not ok:
        raise SystemExit(f"4-bit adapter parity failed before timing: {worst}")
    set_bytes = sum(algorithmic_bytes_q4(s.K, s.N, s.r, 0) for s in HEAD_SPECS)
    copies = int(np.ceil(4 * l2 / set_bytes)) + 1
    sets = [q4] + [{n: _clone_layer(slim, q4[n], dev) for n in names} for _ in range(copies - 1)]
    Y = {(n, M): torch.empty(M, q4[n].N, dtype=torch.bfloat16, device=dev) for n in names for M in DECODE_M}
    wsp = torch.zeros(max(max(q4[n].workspace_bytes(max(DECODE_M)) for n in names), 16), dtype=torch.uint8,
                      device=dev)
    out = {"parity": {"rel_fro": worst[0], "max_abs_rel": worst[1], "pass": bool(ok),
                      "checked": "26 sampled output rows of every layer at M = 1 and 16 vs the fp64 oracle's "
                                 "4-bit adapter forward"},
           "copies": copies, "per_m": {}, "per_layer_us": {}}
    for M in DECODE_M:
        def fn(M=M):
            for s in sets:
                for n in names:
                    slim.linear(s[n], Xd[n][:M], Y[(n, M)], wsp, stream=stream)
        g = _capture(torch, fn, stream)
        med, p10, p90 = _pcts(_time_replays(torch, [g], stream, reps=100))
        b = copies * sum(algorithmic_bytes_q4(s.K, s.N, s.r, M) for s in HEAD_SPECS)
        gbs = b / (med / 1e3) / 1e9
        us = med * 1e3 / copies
        out["per_m"][str(M)] = {"us_per_set": round(us, 2), "GB/s": round(gbs, 1),
                                "frac_hbm": round(gbs / hbm_peak, 4),
                                "speedup_vs_bf16_adapter": round(per_m_bf16[str(M)]["us_per_set"] / us, 3),
                                "launches_per_call": [q4[n].launches(M) for n in names]}
        del g
    for spec in HEAD_SPECS:
        n = spec.name
        lb = algorithmic_bytes_q4(spec.K, spec.N, spec.r, 0)
        nc = min(int(np.ceil(4 * l2 / lb)) + 1, 80)
        cl = [q4[n]] + [_clone_layer(slim, q4[n], dev) for _ in range(nc - 1)]
        ent = {}
        for M in DECODE_M:
            def fn1(M=M, cl=cl, n=n):
                for c in cl:
                    slim.linear(c, Xd[n][:M], Y[(n, M)], wsp, stream=stream)
            g = _capture(torch, fn1, stream)
            ent[str(M)] = round(float(np.median(_time_replays(torch, [g], stream, reps=30))) * 1e3 / nc, 2)
            del g
        out["per_layer_us"][n] = ent
        del cl
        torch.cuda.empty_cache()
    del sets, q4
    torch.cuda.empty_cache()
    return out


def dense_baseline(torch, dev, stream, l2, per_m, pre):
    """torch.matmul(X, W^T) on dense bf16 weights of the six shapes (one copy of
    the set, 1.9 GB, so decode reads from HBM), without and with the adapter
    as two extra matmuls; times per set and slim's speedup."""
    out = {}
    g = torch.Generator(device="cpu").manual_seed(7)
    Ws = [(torch.randn(s.N, s.K, generator=g) * 0.015).to(torch.bfloat16).to(dev) for s in HEAD_SPECS]
    Ls = [(torch.randn(s.K, s.r, generator=g) * 0.01).to(torch.bfloat16).to(dev) for s in HEAD_SPECS]
    Rs = [(torch.randn(s.r, s.N, generator=g) * 0.01).to(torch.bfloat16).to(dev) for s in HEAD_SPECS]
    for M in DECODE_M + PREFILL_M:
        Xs = [torch.randn(M, s.K, device=dev, dtype=torch.bfloat16) for s in HEAD_SPECS]
        for with_ad in (False, True):
            def fn(Xs=Xs, with_ad=with_ad):
                for X, W, L, R in zip(Xs, Ws, Ls, Rs):
                    y = torch.matmul(X, W.t())
                    if with_ad:
                        y = y + torch.matmul(torch.matmul(X, L), R)
            gr = _capture(torch, fn, stream)
            us = float(np.median(_time_replays(torch, [gr], stream, reps=20 if M <= 16 else 10))) * 1e3
            key = f"M{M}" + ("+adapter" if with_ad else "")
            ent = {"us_per_set": round(us, 1)}
            slim_us = per_m[str(M)]["us_per_set"] if M in DECODE_M else pre[str(M)]["us_per_set"]
            ent["slim_speedup"] = round(us / slim_us, 3)
            out[key] = ent
            del gr
        del Xs
    del Ws, Ls, Rs
    torch.cuda.empty_cache()
    return out


def run_q7(torch, slim, dev, stream, hbm_peak):
    """7B q_proj (K = N = 4096, r = 128) decode sweep, 60 rotating copies."""
    spec = Q7_SPEC
    li = make_layer(spec, max(Q7_M))
    base = slim.pack(_to_dev(li.W, dev), _to_dev(li.L, dev), _to_dev(li.R, dev))
    X = _to_dev(li.X, dev)
    cl = [base] + [_clone_layer(slim, base, dev) for _ in range(59)]
    wsp = torch.zeros(max(base.workspace_bytes(max(Q7_M)), 16), dtype=torch.uint8, device=dev)
    out = {}
    for M in Q7_M:
        Y = torch.empty(M, spec.N, dtype=torch.bfloat16, device=dev)

        def fn(M=M, Y=Y):
            for c in cl:
                slim.linear(c, X[:M], Y, wsp, stream=stream)
        g = _capture(torch, fn, stream)
        med, p10, p90 = _pcts(_time_replays(torch, [g], stream, reps=100))
        us = med * 1e3 / len(cl)
        gbs = algorithmic_bytes(spec.K, spec.N, spec.r, M) / (us * 1e-6) / 1e9
        out[str(M)] = {"us_per_call": round(us, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4),
                       "launches": base.launches(M)}
        del g
    del cl
    torch.cuda.empty_cache()
    return out


def run_mlp7(torch, slim, dev, stream, tc_peak):
    """7B MLP up (4096 -> 11008) and down (11008 -> 4096) at M = 2048."""
    M = MLP7_M
    out, lays = {}, []
    for spec in MLP7_SPECS:
        li = make_layer(spec, M)
        lay = slim.pack(_to_dev(li.W, dev), _to_dev(li.L, dev), _to_dev(li.R, dev))
        lays.append((spec, lay, _to_dev(li.X, dev), torch.empty(M, spec.N, dtype=torch.bfloat16, device=dev)))
    wsp = torch.zeros(max(l.workspace_bytes(M) for _, l, _, _ in lays), dtype=torch.uint8, device=dev)
    tot_fl = tot_us = 0.0
    for spec, lay, X, Y in lays:
        def fn(lay=lay, X=X, Y=Y):
            slim.linear(lay, X, Y, wsp, stream=stream)
        g = _capture(torch, fn, stream)
        us = float(np.median(_time_replays(torch, [g], stream, reps=50))) * 1e3
        fl = kept_flops(spec.K, spec.N, spec.r, M)
        out[spec.name] = {"us": round(us, 1), "TFLOP/s": round(fl / (us * 1e-6) / 1e12, 1),
                          "frac_tensor": round(fl / (us * 1e-6) / 1e12 / tc_peak, 4), "launches": lay.launches(M)}
        tot_fl += fl
        tot_us += us
        del g
    out["pair"] = {"TFLOP/s": round(tot_fl / (tot_us * 1e-6) / 1e12, 1),
                   "frac_tensor": round(tot_fl / (tot_us * 1e-6) / 1e12 / tc_peak, 4)}
    del lays
    torch.cuda.empty_cache()
    return out


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

    Mmax = max(BLOCK_M)
    lis = {s.name.split(".")[1]: make_layer(s, Mmax) for s in BLOCK_SPECS}
    W = {k: _to_dev(v.W, dev) for k, v in lis.items()}
    Ld = {k: _to_dev(v.L, dev) for k, v in lis.items()}
    Rd = {k: _to_dev(v.R, dev) for k, v in lis.items()}
    X4 = _to_dev(lis["q"].X, dev)          # [Mmax][4096]: the input of q, k, v, o, gate, up
    X11 = _to_dev(lis["down"].X, dev)      # [Mmax][11008]: the input of down
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
    seps = [sep0] + [{k: _clone_layer(slim, v, dev) for k, v in sep0.items()} for _ in range(copies - 1)]
    fuseds = [fused0] + [{"qkv": _clone_layer(slim, fused0["qkv"], dev), "o": c["o"],
                          "gateup": _clone_layer(slim, fused0["gateup"], dev), "down": c["down"]} for c in seps[1:]]
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
                                     ("up", Yg, 11008, lis["up"], lis["q"].X),
                                     ("down", Yd, 0, lis["down"], lis["down"].X)):
            vals, meta, sc = oracle.pack_layer(np.ascontiguousarray(li.W[rows]))
            ref = oracle.forward(vals, meta, sc, li.L, np.ascontiguousarray(li.R[:, rows]), Xb[:16])
            e = oracle.errors(Y.float().cpu().numpy()[:, off + rows], ref)
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        parity = {"rel_fro": worst[0], "max_abs_rel": worst[1], "pass": bool(worst[0] <= oracle.REL_FRO_TOL and
                                                                             worst[1] <= oracle.MAX_ABS_TOL)}
        if not parity["pass"]:
            raise SystemExit(f"parity check failed before timing: {parity}")

    stream = torch.cuda.Stream(device=dev)
    hbm_peak, tc_peak, _, peak_kind = load_peaks()
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
                g = _capture(torch, fn, stream)
                reps = 10 if M <= 16 else 5
                res[tag] = float(np.median(_time_replays(torch, [g], stream, reps=reps,
                                                         warmup=max(3, args.warmup)))) * 1e3 / copies
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["slim", "reference"], default="slim")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["headline", "block"], default="headline",
                    help="headline: the six 70B-shaped linears, decode value + prefill (default); "
                         "block: the 7 linears of a 7B decoder block, separate and fused, M in {1..4096}")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "block":
        run_block(args)
    else:
        run_headline(args)


if __name__ == "__main__":
    main()
