"""The benchmark's multi-rank path on CPU: two gloo ranks on 127.0.0.1.

With N GPUs every rank decodes its own sequences (the path splits by
sequence and needs no collective), and the job time is the slowest rank's.
These tests run the aggregation that bench.py uses, and the per-rank
workload recipe, in world_size-2 process groups."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) * 10 ms for 100 steps of 1 MB each
        ms = bench.max_over_ranks(torch, (rank + 1) * 10.0, world)
        gbs = bench.job_throughput(1e6, ms, 100, world)
        # every rank builds a replica of the same shape from its own seed
        os.environ["RANK"] = str(rank)
        w = bench.make_workload("tiny", None, rank, nthreads=1)
        q.put((rank, ms, gbs, w.q.shape, int(w.q[0, 0, 0])))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, gbs, shape, _ in res:
        assert ms == pytest.approx(20.0)            # max over ranks
        # 2 ranks x 1 MB per step over 0.2 ms per step
        assert gbs == pytest.approx(2 * 1e6 / (20.0e-3 / 100) / 1e9)
        assert tuple(shape) == (1, 8, 64)
    # the replicas decode different sequences
    assert res[0][4] != res[1][4]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import torch

    import bench
    assert bench.max_over_ranks(torch, 12.5, 1) == 12.5
    assert bench.job_throughput(2e6, 10.0, 10, 1) == pytest.approx(2e6 / 1e-3 / 1e9)
