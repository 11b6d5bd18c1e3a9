"""Multi-rank plumbing of the benchmark on the CPU (gloo, world size 2).

The decode path shards over independent (sequence, layer) problems, so ranks
run replicas with no exchange on the data path; the only cross-rank steps are
the barrier around the timed region and the max over ranks of the elapsed
time.  These run here with the gloo backend, no GPU involved.
"""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        dist.barrier()
        mine = 0.5 + rank                                  # rank 1 is the slow one
        slowest = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        q.put((rank, slowest, bench.replica_value(world, 10, slowest)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [1.5, 1.5]          # every rank sees the slowest time
    assert all(abs(g[2] - 2 * 10 / 1.5) < 1e-12 for g in got)   # units of both replicas / that time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(0.25, None, torch.device("cpu")) == 0.25
    assert bench.replica_value(1, 8, 0.5) == 16.0


def test_reference_arm_prints_nothing_on_other_ranks():
    class A:
        steps, warmup, gpus = 1, 0, 2
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(A(), bench.synth.WORKLOADS[1], rank=1)
    assert buf.getvalue() == ""
