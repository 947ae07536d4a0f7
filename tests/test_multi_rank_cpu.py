"""The N > 1 path of bench.py on CPU: gloo ranks, no GPU.

The decode path shards without any exchange (independent replicas over
sequences), so the only multi-rank logic is the plumbing around it: process
group set-up, the barrier around the timed region, the max over ranks of the
device time, and the reference arm that only rank 0 runs.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, queue) -> None:
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    w, r, local = bench.dist_setup()
    backend = dist.get_backend()
    bench.barrier(w)
    # each rank reports a different device time; every rank must see the slowest
    m = bench.max_over_ranks(1.5 + rank, w, torch.device("cpu"))
    bench.barrier(w)
    dist.destroy_process_group()
    queue.put((rank, w, r, local, backend, m))


def test_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(i, world, port, queue)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(queue.get(timeout=10) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    for rank, w, r, local, backend, m in got:
        assert (w, r, local, backend) == (world, rank, rank, "gloo")
        assert m == 1.5 + (world - 1)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["config"]["workload"] == "tiny"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
