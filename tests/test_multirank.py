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


def _sharded_worker(rank, world, port, q_out):
    """One rank of a sequence-parallel decode on CPU: the partial over this
    rank's slice comes from the fp64 oracle, the merge is the log-sum-exp
    formula written out in numpy; the packing, the one all-gather and the
    unpacking of the gathered parts are the package's own code."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from split_kv_decode_attn_b200 import sharded
    from split_kv_decode_attn_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.make_problem(3, 8, 2, 64, 300, seed=77, seqlens=[300, 120, 0])
        lo, hi = sharded.shard_bounds(w.max_len, world, rank)
        sl_shard = sharded.shard_lengths(w.seqlens, lo, hi)
        k_shard = np.ascontiguousarray(w.k[:, :, lo:hi])
        v_shard = np.ascontiguousarray(w.v[:, :, lo:hi])

        def partial(q, k, v, seqlens):
            o, lse = oracle.decode(q, k, v, w.scale, seqlens=seqlens, nthreads=1)
            buf = torch.full((sharded.packed_floats(w.B, w.Hq, w.D),), float("nan"),
                             dtype=torch.float64)
            po, pl = sharded.unpack(buf, w.B, w.Hq, w.D)
            po.copy_(torch.from_numpy(o))
            pl.copy_(torch.from_numpy(lse))
            return buf

        def merge(parts, B, Hq, D):
            assert tuple(parts.shape) == (world, sharded.packed_floats(B, Hq, D))
            o_all, lse_all = sharded.unpack(parts, B, Hq, D)
            o_all, lse_all = o_all.numpy(), lse_all.numpy()
            m = lse_all.max(axis=0)
            with np.errstate(invalid="ignore"):
                wgt = np.where(np.isneginf(lse_all), 0.0, np.exp(lse_all - m))
            tot = wgt.sum(axis=0)
            out = np.where(tot[..., None] > 0,
                           (wgt[..., None] * o_all).sum(axis=0) / np.where(tot > 0, tot, 1)[..., None], 0.0)
            lse = np.where(tot > 0, m + np.log(np.where(tot > 0, tot, 1)), -np.inf)
            return out, lse

        out, lse = sharded.decode_sequence_sharded(w.q, k_shard, v_shard, np.array(sl_shard, np.int32),
                                                   partial=partial, merge=merge)
        ref, ref_lse = oracle.decode(w.q, w.k, w.v, w.scale, seqlens=w.seqlens, nthreads=1)
        q_out.put((rank, float(np.max(np.abs(out - ref))),
                   bool(np.all(np.isneginf(lse[2]))),
                   float(np.max(np.abs(lse[:2] - ref_lse[:2])))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharded_decode_orchestration(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = [q.get(timeout=10) for _ in range(world)]
    for rank, err, empty_ok, lse_err in res:
        assert err < 1e-12 and lse_err < 1e-12 and empty_ok, (rank, err, lse_err)


def test_packed_partial_layout():
    """One part is O rows then lse values, padded to 64 floats; unpack gives
    views of one part or of R gathered parts."""
    sys.path.insert(0, ROOT)
    import torch

    from split_kv_decode_attn_b200 import sharded
    for B, Hq, D in ((1, 1, 64), (3, 8, 64), (1, 64, 128), (2, 6, 128)):
        P = sharded.packed_floats(B, Hq, D)
        rows = B * Hq
        assert P % 64 == 0 and rows * (D + 1) <= P < rows * (D + 1) + 64
        parts = torch.arange(3 * P, dtype=torch.float32).reshape(3, P)
        o, lse = sharded.unpack(parts, B, Hq, D)
        assert o.shape == (3, B, Hq, D) and lse.shape == (3, B, Hq)
        assert o[2, B - 1, Hq - 1, D - 1] == 2 * P + rows * D - 1
        assert lse[1, 0, 0] == P + rows * D and lse[1, B - 1, Hq - 1] == P + rows * D + rows - 1
        o1, l1 = sharded.unpack(parts[1], B, Hq, D)
        assert o1.data_ptr() == parts[1].data_ptr() and torch.equal(l1, lse[1])


def test_shard_bounds_cover_the_history_once():
    sys.path.insert(0, ROOT)
    from split_kv_decode_attn_b200 import sharded
    for total in (0, 1, 7, 300, 4096):
        for world in (1, 2, 3, 8):
            ranges = [sharded.shard_bounds(total, world, r) for r in range(world)]
            covered = [t for lo, hi in ranges for t in range(lo, hi)]
            assert covered == list(range(total))
    assert sharded.shard_lengths([300, 120, 0], 100, 200) == [100, 20, 0]
