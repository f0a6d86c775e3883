"""Sequence-parallel decode: every rank holds a contiguous slice of each
sequence's cached history.

Each rank computes the exact attention over its own slice (fd_decode_partial:
fp32 output plus log-sum-exp).  The R partial results are all-gathered (one
NCCL all-gather of B*Hq*(D+1) floats per rank) and merged on every rank by
fd_combine, the same log-sum-exp reduction that merges the splits of one GPU
("What is Flash-Decoding, and when does it speed up LLMs?", section "Why
decode needs a different schedule").  The result equals attention over the
whole history on every rank.

The compute steps are arguments so that the orchestration (slice bounds,
gather order) can also be driven by other implementations; by default they
are the CUDA library's.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence


def shard_bounds(total_len: int, world: int, rank: int):
    """Token range [lo, hi) of `rank`'s slice when `total_len` cached tokens are
    cut into `world` contiguous slices of ceil(total_len / world) tokens."""
    per = -(-total_len // world)
    lo = min(rank * per, total_len)
    hi = min(lo + per, total_len)
    return lo, hi


def shard_lengths(seqlens: Sequence[int], lo: int, hi: int):
    """Valid tokens of each sequence inside the slice [lo, hi)."""
    return [max(0, min(int(n), hi) - lo) for n in seqlens]


def local_partial(q, k_shard, v_shard, seqlens_shard=None, *, block_table=None, scale=None,
                  num_splits=None, kv_layout: int = 0, stream=None):
    """fd_decode_partial on this rank's slice; returns (o_f32 [B, Hq, D], lse [B, Hq])."""
    import torch

    import split_kv_decode_attn_b200 as fd
    fd._check_decode_args(q, k_shard, v_shard, seqlens_shard, block_table, kv_layout, None,
                          None, None, None)
    B, Hq, D = q.shape
    if block_table is None:
        if kv_layout == fd.FD_LAYOUT_HND:
            _, Hkv, L, _ = k_shard.shape
        else:
            _, L, Hkv, _ = k_shard.shape
        prob = fd.make_problem(B, Hq, Hkv, D, L, kv_layout=kv_layout)
        bs = 0
    else:
        if kv_layout == fd.FD_LAYOUT_HND:
            nb, Hkv, bs, _ = k_shard.shape
        else:
            nb, bs, Hkv, _ = k_shard.shape
        L = block_table.shape[1] * bs
        prob = fd.make_problem(B, Hq, Hkv, D, L, bs, nb, block_table.shape[1], kv_layout)
    scale = 1.0 / D ** 0.5 if scale is None else scale
    if num_splits is None:
        num_splits = fd.fd_plan(B, Hq, Hkv, D, L, bs)
    o = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    nbytes = fd.fd_workspace_bytes(B, Hq, D, num_splits)
    ws = torch.empty(max(nbytes, 4) // 4, dtype=torch.float32, device=q.device)
    st = fd.fd_decode_partial(prob, q, k_shard, v_shard, seqlens_shard, block_table, scale,
                              num_splits, o, lse, ws, nbytes, stream)
    if st != fd.FD_OK:
        raise fd.FdError(st, "fd_decode_partial")
    return o, lse


def combine(o_all, lse_all, stream=None):
    """fd_combine of gathered partials o_all [R, B, Hq, D], lse_all [R, B, Hq]."""
    import torch

    import split_kv_decode_attn_b200 as fd
    R, B, Hq, D = o_all.shape
    if o_all.dtype != torch.float32 or lse_all.dtype != torch.float32:
        raise ValueError("combine: o_all and lse_all must be float32")
    if tuple(lse_all.shape) != (R, B, Hq):
        raise ValueError(f"combine: lse_all shape {tuple(lse_all.shape)}, expected {(R, B, Hq)}")
    if not (o_all.is_cuda and lse_all.device == o_all.device):
        raise ValueError("combine: o_all and lse_all must be on one CUDA device")
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=o_all.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=o_all.device)
    st = fd.fd_combine(R, B, Hq, D, o_all.contiguous(), lse_all.contiguous(), out, lse, stream)
    if st != fd.FD_OK:
        raise fd.FdError(st, "fd_combine")
    return out, lse


def decode_sequence_sharded(q, k_shard, v_shard, seqlens_shard=None, *, group=None,
                            partial: Optional[Callable] = None,
                            merge: Optional[Callable] = None, **kw):
    """Attention over the whole history, from this rank's slice.

    Every rank passes the same q and its own k/v slice (and the valid
    tokens of each sequence inside it).  Returns (out, lse) for the whole
    history on every rank.  `partial(q, k, v, seqlens, **kw)` and
    `merge(o_all, lse_all)` default to the CUDA library."""
    import torch
    import torch.distributed as dist
    partial = partial or local_partial
    merge = merge or combine
    o, lse = partial(q, k_shard, v_shard, seqlens_shard, **kw)
    world = dist.get_world_size(group)
    o_list = [torch.empty_like(o) for _ in range(world)]
    l_list = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(o_list, o.contiguous(), group=group)
    dist.all_gather(l_list, lse.contiguous(), group=group)
    return merge(torch.stack(o_list), torch.stack(l_list))
