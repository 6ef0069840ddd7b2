"""The multi-rank host logic of bench.py on CPU: world size 2 over gloo (127.0.0.1).

Each rank runs its own independent batch (replicas, weak scaling): the step time reported is
the slowest rank's, the value is every rank's tokens over that time, and only rank 0 prints.
"""
import io
import os
import contextlib

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_setup(None)
        ms = 10.0 * (rank + 1)                 # rank 1 is the slow one
        slow = bench.slowest(ms, dist, "cpu")
        rate = bench.throughput(8, w, slow)
        # the reference arm: rank 0 alone runs and prints
        class A:
            gpus, steps, warmup = w, 1, 1
        wl = bench.W.make_workload(0, lengths=[64], n_sparse=1)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(A, wl)
        q.put((rank, w, r, slow, rate, buf.getvalue()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_rank0_prints():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, w, r, slow, rate, out in res:
        assert (w, r) == (2, rank)
        assert slow == pytest.approx(20.0)
        assert rate == pytest.approx(2 * 8 / 0.020)
    assert '"impl": "reference"' in res[0][5]
    assert res[1][5] == ""


def test_single_rank_is_its_own_slowest():
    assert bench.slowest(3.5) == 3.5
    assert bench.throughput(8, 1, 2.0) == pytest.approx(4000.0)
