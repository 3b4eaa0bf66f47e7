"""Multi-process host logic of bench.py (replicas, one process per GPU) on
CPU: two gloo ranks check the barrier, the max/sum reductions and the
whole-job rate (units of all ranks over the slowest rank's time)."""
import os
import socket
import sys
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, str(ROOT))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = 10.0 * (rank + 1)                  # rank r took 10(r+1) ms for 100(r+1) tokens
        units = 100.0 * (rank + 1)
        res = (bench.max_over_ranks(ms, world), bench.sum_over_ranks(units, world),
               bench.job_rate(units, ms, world))
        out.put((rank, res))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_reductions_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get() for _ in range(world))
    for r in range(world):
        mx, sm, rate = got[r]
        assert mx == 20.0                        # slowest rank
        assert sm == 300.0                       # all ranks' tokens
        assert rate == pytest.approx(300.0 / 0.020)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, str(ROOT))
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(7.0, 1) == 7.0
    assert bench.job_rate(50.0, 10.0, 1) == pytest.approx(5000.0)
