"""The bench's multi-rank plumbing with two gloo ranks on CPU (no GPU).

bench.py runs one process per GPU under torchrun; every rank runs the same
replica, timings are reduced with MAX (the slowest rank times the job), the
whole-job value counts the units of all ranks, and only rank 0 prints.
"""
from __future__ import annotations

import datetime
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.rank_env()
        # per-rank timings that differ: rank 1 is slower in the first, rank 0 in the second
        vals = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 3.0], w, "cpu")
        rate = bench.whole_job_rate(100.0, vals[0], w)
        out.put((rank, r, w, lr, vals, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_with_max():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, w, lr, vals, rate in res:
        assert (r, w, lr) == (rank, 2, rank)
        assert vals == [2.0, 5.0, 3.0]            # the slowest rank, element by element
        assert rate == pytest.approx(2 * 100.0 / 2.0e-3)   # both ranks' units over the slowest time


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.whole_job_rate(10.0, 2.0, 1) == pytest.approx(5000.0)


def test_reference_arm_on_a_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
