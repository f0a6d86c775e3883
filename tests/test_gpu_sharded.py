"""Sequence-parallel decode on one GPU: the history is cut into R contiguous
slices; fd_decode_partial runs on each slice, the R results are laid out as an
all-gather would lay them out (stacked, or packed buffers end to end) and
fd_combine / fd_combine_strided merge them.  The slices run one after another
on one device, so nothing waits on anything else; with one GPU per rank the
same partials would be all-gathered instead."""
import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import sharded
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import OnDevice, assert_close, dev_bf16, dev_i32, host_bf16, reference, run_gpu

pytestmark = pytest.mark.gpu


def slice_workload(w, lo, hi):
    """The contiguous cache rows [lo, hi) of every sequence, as a workload."""
    sl = sharded.shard_lengths(w.lengths(), lo, hi)
    return wl.Workload(name="slice", B=w.B, Hq=w.Hq, Hkv=w.Hkv, D=w.D, max_len=hi - lo, q=w.q,
                       k=np.ascontiguousarray(w.k[:, :, lo:hi]),
                       v=np.ascontiguousarray(w.v[:, :, lo:hi]), scale=w.scale,
                       seqlens=np.array(sl, np.int32))


def partial_on_gpu(w, S=None):
    import torch
    d = OnDevice(w)
    S = S or d.plan()
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.D, S)
    ws = torch.empty(max(nbytes, 4) // 4, dtype=torch.float32, device="cuda")
    st = fd.fd_decode_partial(d.problem(), d.q, d.k, d.v, d.seqlens, d.table, w.scale, S, o, lse,
                              ws, nbytes, None)
    assert st == fd.FD_OK, fd.fd_status_string(st)
    return o, lse


@pytest.mark.parametrize("S", [1, 4, 24])
def test_partial_is_exact_attention_in_fp32(cuda_device, S):
    import torch
    w = wl.make_problem(3, 32, 8, 128, 3000, seed=90, seqlens=[3000, 17, 0])
    o, lse = partial_on_gpu(w, S)
    torch.cuda.synchronize()
    ref, rl = reference(w)
    got = o.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-3
    gl = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isneginf(gl[2])) and np.all(got[2] == 0)
    assert np.max(np.abs(gl[:2] - rl[:2])) <= 1e-3


@pytest.mark.parametrize("R", [1, 2, 3, 4])
def test_slices_merge_into_whole_history(cuda_device, R):
    import torch
    w = wl.make_problem(4, 64, 8, 128, 8192, seed=91 + R, seqlens=[8192, 5000, 300, 0])
    parts = []
    for r in range(R):
        lo, hi = sharded.shard_bounds(w.max_len, R, r)
        parts.append(partial_on_gpu(slice_workload(w, lo, hi)))
    o_all = torch.stack([p[0] for p in parts])
    l_all = torch.stack([p[1] for p in parts])
    out, lse = sharded.combine(o_all, l_all)
    torch.cuda.synchronize()
    ref, rl = reference(w)
    assert_close(host_bf16(out), lse.cpu().numpy().astype(np.float64), ref, rl, f"R={R}")
    # and agrees with the single-GPU call over the whole history
    whole, wl_, _ = run_gpu(OnDevice(w))
    assert np.max(np.abs(host_bf16(out) - whole)) <= 1e-2
    assert fd.fd_check_device_error() == fd.FD_OK


def test_combine_of_empty_parts_and_bad_arguments(cuda_device):
    import torch
    R, B, Hq, D = 3, 2, 8, 64
    o_all = torch.zeros((R, B, Hq, D), dtype=torch.float32, device="cuda")
    l_all = torch.full((R, B, Hq), float("-inf"), dtype=torch.float32, device="cuda")
    out = torch.full((B, Hq, D), 5.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
    assert fd.fd_combine(R, B, Hq, D, o_all, l_all, out, lse) == fd.FD_OK
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    assert fd.fd_combine(0, B, Hq, D, o_all, l_all, out, lse) == fd.FD_ERR_INVALID_ARGUMENT
    assert fd.fd_combine(R, B, Hq, 96, o_all, l_all, out, lse) == fd.FD_ERR_UNSUPPORTED


def test_paged_slices_merge(cuda_device):
    """Each rank holds whole pages of the history; the slices are paged caches."""
    import torch
    B, Hq, Hkv, D, L, bs, R = 2, 32, 8, 128, 2048, 16, 2
    w = wl.make_problem(B, Hq, Hkv, D, L, seed=95, seqlens=[2048, 1000], block_size=bs)
    parts = []
    for r in range(R):
        lo, hi = sharded.shard_bounds(L, R, r)
        table = np.ascontiguousarray(w.block_table[:, lo // bs:hi // bs])
        sl = np.array(sharded.shard_lengths(w.lengths(), lo, hi), np.int32)
        s = wl.Workload(name="pslice", B=B, Hq=Hq, Hkv=Hkv, D=D, max_len=hi - lo, q=w.q, k=w.k,
                        v=w.v, scale=w.scale, seqlens=sl, block_size=bs, block_table=table)
        parts.append(partial_on_gpu(s))
    out, lse = sharded.combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()
    ref, rl = reference(w)
    assert_close(host_bf16(out), lse.cpu().numpy().astype(np.float64), ref, rl, "paged slices")


@pytest.mark.parametrize("R", [1, 2, 3])
def test_packed_parts_merge_where_they_lie(cuda_device, R):
    """The sequence-parallel exchange format: each slice's partial is written
    by sharded.local_partial straight into its row of one [R, P] buffer (the
    layout an all-gather of the packed buffers produces), and
    fd_combine_strided merges the rows in place.  The result equals the
    merge of the same partials stacked into [R, B, Hq, D] / [R, B, Hq] bit
    for bit, and the fp64 oracle over the whole history."""
    import torch
    B, Hq, Hkv, D, L = 2, 32, 8, 128, 4096
    w = wl.make_problem(B, Hq, Hkv, D, L, seed=96 + R, seqlens=[4096, 1500])
    P = sharded.packed_floats(B, Hq, D)
    parts = torch.full((R, P), float("nan"), dtype=torch.float32, device="cuda")
    for r in range(R):
        lo, hi = sharded.shard_bounds(L, R, r)
        d = OnDevice(slice_workload(w, lo, hi))
        sharded.local_partial(d.q, d.k, d.v, d.seqlens, packed=parts[r])
    out, lse = sharded.combine_packed(parts, B, Hq, D)
    o_all, l_all = sharded.unpack(parts, B, Hq, D)
    out2, lse2 = sharded.combine(o_all.contiguous(), l_all.contiguous())
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    ref, rl = reference(w)
    assert_close(host_bf16(out), lse.cpu().numpy().astype(np.float64), ref, rl, f"packed R={R}")
    # strides that would put a part's rows out of line are refused
    base = parts.data_ptr()
    assert fd.fd_combine_strided(R, B, Hq, D, base, P - 2, base + 4 * B * Hq * D, P, out,
                                 lse) == fd.FD_ERR_INVALID_ARGUMENT
    assert fd.fd_combine_strided(R, B, Hq, D, base, B * Hq * D - 4, base, P, out,
                                 lse) == fd.FD_ERR_INVALID_ARGUMENT
    assert fd.fd_check_device_error() == fd.FD_OK
