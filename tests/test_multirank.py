"""bench.py's multi-process plumbing on CPU (gloo, world size 2).

The path shards as independent replicas (no data exchange), so the only
collectives are the barrier and the max-over-ranks of the timed region.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_decode_30_b200 import workloads as W
    rank_, world_, _ = bench.dist_setup(bench.parse_args([]))
    try:
        assert (rank_, world_) == (rank, world)
        bench.barrier(world)
        elapsed = 10.0 + 5.0 * rank          # a slower rank decides the time
        mx = bench.max_over_ranks(elapsed, world)
        total = bench.sum_over_ranks(1.0, world)
        wl = W.TINY
        inp = W.generate(wl, seed=wl.seed + rank)  # each replica its own batch
        out_q.put((rank, mx, total, float(inp["q"].float().sum())))
    finally:
        dist.destroy_process_group()


def test_replicas_take_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]   # max over ranks on every rank
    assert [r[2] for r in res] == [2.0, 2.0]
    assert res[0][3] != res[1][3]                # replicas draw different inputs


def test_reference_arm_runs_on_rank0_only():
    """Under torchrun with 2 ranks, only rank 0 times the oracle and prints."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
