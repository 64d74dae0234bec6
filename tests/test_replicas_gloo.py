"""The N > 1 plumbing of bench.py, exercised on CPU with gloo ranks.

The forward does not shard (replicas only: every rank runs the whole
workload on its own GPU, no collective on the data path), so what N > 1
adds is host logic: the ranks join one process group, the step time is the
slowest rank's (an all-reduce MAX), and only rank 0 prints.  These tests run
that logic with world size 2 on the gloo backend, and the reference arm
(the oracle on rank 0's host cores) under torchrun with two ranks.
"""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="host-only (gloo) path of the rank plumbing")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2",
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    ws, r, _ = bench.dist_setup(None)
    slowest = bench.max_over_ranks(10.0 + 5.0 * r, ws)   # rank 1 is the slow one
    bench.barrier(ws)
    q.put((r, ws, dist.get_backend(), slowest))
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2, "gloo", 15.0), (1, 2, "gloo", 15.0)]


def test_reference_arm_under_torchrun_prints_one_line():
    """Rank 0 times the oracle and prints the JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
