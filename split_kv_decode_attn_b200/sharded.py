"""Sequence-parallel decode: every rank holds a contiguous slice of each
sequence's cached history.

Each rank computes the exact attention over its own slice (fd_decode_partial:
fp32 output plus log-sum-exp), written straight into one packed buffer of
B*Hq*(D+1) floats (padded to 256 bytes): the output rows, then their lse
values.  One all-gather (all_gather_into_tensor) lays the R packed buffers end
to end, and fd_combine_strided merges them where they lie, on every rank,
with the same log-sum-exp reduction that merges the splits of one GPU ("What
is Flash-Decoding, and when does it speed up LLMs?", section "Why decode needs
a different schedule").  The result equals attention over the whole history
on every rank.

The compute steps are arguments so that the orchestration (slice bounds,
packing, gather order) can also be driven by other implementations; by
default they are the CUDA library's.
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


def packed_floats(B: int, Hq: int, D: int) -> int:
    """Floats of one rank's packed partial: O [B*Hq*D], then lse [B*Hq], then
    padding to a multiple of 64 floats, so that every part of a gathered
    buffer starts 256-byte aligned."""
    rows = B * Hq
    return -(-(rows * D + rows) // 64) * 64


def unpack(buf, B: int, Hq: int, D: int):
    """Views (o [..., B, Hq, D], lse [..., B, Hq]) of packed buffers
    [..., packed_floats(B, Hq, D)] (one part or R gathered parts)."""
    rows = B * Hq
    lead = tuple(buf.shape[:-1])
    return (buf[..., :rows * D].reshape(lead + (B, Hq, D)),
            buf[..., rows * D:rows * D + rows].reshape(lead + (B, Hq)))


def local_partial(q, k_shard, v_shard, seqlens_shard=None, *, block_table=None, scale=None,
                  num_splits=None, kv_layout: int = 0, stream=None, packed=None):
    """fd_decode_partial on this rank's slice, written into `packed` (a float32
    CUDA tensor of packed_floats(B, Hq, D), allocated when None).  Returns the
    packed tensor.  Temporaries are allocated on the stream the kernels run
    on, so that torch's allocator does not hand their memory to other work
    while the kernels still use it."""
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
    P = packed_floats(B, Hq, D)
    if packed is not None:
        if (packed.dtype != torch.float32 or tuple(packed.shape) != (P,) or
                not packed.is_contiguous() or packed.device != q.device):
            raise ValueError(f"packed: expected a contiguous float32 tensor of {P} floats on "
                             f"{q.device}")
    torch_stream = (stream if isinstance(stream, torch.cuda.Stream) else
                    torch.cuda.current_stream(q.device) if stream is None else
                    torch.cuda.ExternalStream(stream, device=q.device))
    nbytes = fd.fd_workspace_bytes(B, Hq, D, num_splits)
    with torch.cuda.stream(torch_stream):
        if packed is None:
            packed = torch.empty(P, dtype=torch.float32, device=q.device)
        ws = torch.empty(max(nbytes, 4) // 4, dtype=torch.float32, device=q.device)
    o, lse = unpack(packed, B, Hq, D)
    st = fd.fd_decode_partial(prob, q, k_shard, v_shard, seqlens_shard, block_table, scale,
                              num_splits, o, lse, ws, nbytes, torch_stream.cuda_stream)
    if st != fd.FD_OK:
        raise fd.FdError(st, "fd_decode_partial")
    return packed


def combine_packed(parts, B: int, Hq: int, D: int, stream=None):
    """fd_combine_strided over R gathered packed partials parts
    [R, packed_floats(B, Hq, D)] (float32, contiguous, one CUDA device),
    merged where they lie.  Returns (out [B, Hq, D] bf16, lse [B, Hq])."""
    import torch

    import split_kv_decode_attn_b200 as fd
    P = packed_floats(B, Hq, D)
    if parts.dtype != torch.float32:
        raise ValueError("combine_packed: parts must be float32")
    if parts.dim() != 2 or parts.shape[1] != P:
        raise ValueError(f"combine_packed: parts shape {tuple(parts.shape)}, expected [R, {P}]")
    if not parts.is_contiguous():
        raise ValueError("combine_packed: parts must be contiguous")
    if not parts.is_cuda:
        raise ValueError("combine_packed: parts must be on a CUDA device")
    R = parts.shape[0]
    torch_stream = (stream if isinstance(stream, torch.cuda.Stream) else
                    torch.cuda.current_stream(parts.device) if stream is None else
                    torch.cuda.ExternalStream(stream, device=parts.device))
    with torch.cuda.stream(torch_stream):
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=parts.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=parts.device)
    rows = B * Hq
    base = parts.data_ptr()
    st = fd.fd_combine_strided(R, B, Hq, D, base, P, base + 4 * rows * D, P, out, lse,
                               torch_stream.cuda_stream)
    if st != fd.FD_OK:
        raise fd.FdError(st, "fd_combine_strided")
    return out, lse


def combine(o_all, lse_all, stream=None):
    """fd_combine of stacked partials o_all [R, B, Hq, D], lse_all [R, B, Hq]."""
    import torch

    import split_kv_decode_attn_b200 as fd
    R, B, Hq, D = o_all.shape
    if o_all.dtype != torch.float32 or lse_all.dtype != torch.float32:
        raise ValueError("combine: o_all and lse_all must be float32")
    if tuple(lse_all.shape) != (R, B, Hq):
        raise ValueError(f"combine: lse_all shape {tuple(lse_all.shape)}, expected {(R, B, Hq)}")
    if not (o_all.is_cuda and lse_all.device == o_all.device):
        raise ValueError("combine: o_all and lse_all must be on one CUDA device")
    if not (o_all.is_contiguous() and lse_all.is_contiguous()):
        raise ValueError("combine: o_all and lse_all must be contiguous")
    torch_stream = (stream if isinstance(stream, torch.cuda.Stream) else
                    torch.cuda.current_stream(o_all.device) if stream is None else
                    torch.cuda.ExternalStream(stream, device=o_all.device))
    with torch.cuda.stream(torch_stream):
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=o_all.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=o_all.device)
    st = fd.fd_combine(R, B, Hq, D, o_all, lse_all, out, lse, torch_stream.cuda_stream)
    if st != fd.FD_OK:
        raise fd.FdError(st, "fd_combine")
    return out, lse


def decode_sequence_sharded(q, k_shard, v_shard, seqlens_shard=None, *, group=None,
                            partial: Optional[Callable] = None,
                            merge: Optional[Callable] = None, **kw):
    """Attention over the whole history, from this rank's slice.

    Every rank passes the same q and its own k/v slice (and the valid
    tokens of each sequence inside it).  Returns (out, lse) for the whole
    history on every rank.

    partial(q, k, v, seqlens, **kw) returns this rank's packed partial (a
    1-D float32 tensor of packed_floats(B, Hq, D)); merge(parts, B, Hq, D)
    merges the gathered [R, packed_floats] tensor.  Both default to the CUDA
    library (local_partial, combine_packed).  The exchange is one
    all_gather_into_tensor of the packed buffers."""
    import torch
    import torch.distributed as dist
    partial = partial or local_partial
    merge = merge or combine_packed
    B, Hq, D = q.shape
    send = partial(q, k_shard, v_shard, seqlens_shard, **kw)
    world = dist.get_world_size(group)
    parts = torch.empty(world * send.numel(), dtype=send.dtype, device=send.device)
    dist.all_gather_into_tensor(parts, send, group=group)   # the parts end to end
    return merge(parts.view(world, send.numel()), B, Hq, D)
