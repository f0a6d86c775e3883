"""Shared helpers of the GPU tests: move a seeded workload to the device, run
fd_decode through the C ABI, compute the fp64 oracle on the same bf16 bytes,
and compare with the stated tolerances.

Tolerances (same for every config):
  out: |out_gpu - O_ref| <= 1e-2 where |O_ref| < 4.  bf16 rounding alone can
       reach half an ulp, which exceeds 1e-2 once |O_ref| >= 4; there the
       bound is half an ulp of O_ref plus 2e-3.
  lse: |lse_gpu - lse_ref| <= 1e-3, and -inf exactly where the sequence is
       empty.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle
import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import workloads as wl

OUT_TOL = 1e-2
LSE_TOL = 1e-3


def torch():
    import torch as _t
    return _t


def dev_bf16(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(t.bfloat16)


def dev_i32(a):
    t = torch()
    return None if a is None else t.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_u8(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def host_bf16(x) -> np.ndarray:
    t = torch()
    return wl.bf16_bits_to_f64(x.view(t.int16).cpu().numpy().view(np.uint16))


class OnDevice:
    """Device copies of a workload's tensors."""

    def __init__(self, w: wl.Workload, fp8_mma: int = 0):
        self.w = w
        self.fp8_mma = fp8_mma
        self.q = dev_bf16(w.q)
        up = dev_bf16 if w.kv_dtype == "bf16" else dev_u8
        self.k = up(w.k)
        self.v = up(w.v)
        self.seqlens = dev_i32(w.seqlens)
        self.table = dev_i32(w.block_table)

    def problem(self):
        w = self.w
        return fd.make_problem(w.B, w.Hq, w.Hkv, w.D, w.max_len, w.block_size, w.num_blocks,
                               w.max_blocks_per_seq, w.kv_layout, w.kv_dtype_code, w.k_scale,
                               w.v_scale, self.fp8_mma)

    def plan(self) -> int:
        """The split count the benchmark uses: fd_plan_problem over the whole
        problem, with the lengths when they are known."""
        s = fd.fd_plan_problem(0, self.problem(), self.w.seqlens)
        assert s >= 1, fd.fd_status_string(s)
        return s

    def run(self, num_splits=None, with_lse=True, stream=None):
        """fd_decode through the C ABI.  Returns (out bf16 tensor, lse tensor|None, S)."""
        t = torch()
        w = self.w
        S = self.plan() if num_splits is None else num_splits
        out = t.empty((w.B, w.Hq, w.D), dtype=t.bfloat16, device="cuda")
        lse = t.empty((w.B, w.Hq), dtype=t.float32, device="cuda") if with_lse else None
        nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.D, S)
        ws = t.empty(max(nbytes, 4) // 4, dtype=t.float32, device="cuda")
        st = fd.fd_decode(self.problem(), self.q, self.k, self.v, self.seqlens, self.table,
                          w.scale, S, out, lse, ws, nbytes, stream)
        assert st == fd.FD_OK, fd.fd_status_string(st)
        return out, lse, S


def run_gpu(d: OnDevice, num_splits=None):
    torch().cuda.synchronize()
    out, lse, S = d.run(num_splits)
    torch().cuda.synchronize()
    assert fd.fd_check_device_error() == fd.FD_OK
    return host_bf16(out), lse.cpu().numpy().astype(np.float64), S


def reference(w: wl.Workload, groups=None, nthreads=None):
    """fp64 oracle on the workload's bf16 bytes.

    groups: iterable of (b, kv_head) to compute, or None for all.  Rows not
    computed are NaN.  Paged caches are gathered to logical token order
    first (the oracle only sees logical K/V)."""
    nthreads = nthreads or os.cpu_count() or 1
    if groups is None and not w.paged and w.layout == "HND" and w.kv_dtype == "bf16":
        return oracle.decode(w.q, w.k, w.v, w.scale, seqlens=w.seqlens, nthreads=nthreads)
    if groups is None:
        groups = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    out = np.full((w.B, w.Hq, w.D), np.nan)
    lse = np.full((w.B, w.Hq), np.nan)
    G = w.G

    def one(bh):
        b, h = bh
        if w.kv_dtype == "bf16":
            k, v = w.logical_kv(b, h)
            o, l = oracle.attend(w.q[b, h * G:(h + 1) * G], np.ascontiguousarray(k),
                                 np.ascontiguousarray(v), w.scale)
        else:  # dequantised fp8 values in fp64
            k, v = w.logical_kv_f64(b, h)
            o, l = oracle.attend_f64(wl.bf16_bits_to_f64(w.q[b, h * G:(h + 1) * G]), k, v,
                                     float(np.float32(w.scale)))
        return b, h, o, l

    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        for b, h, o, l in ex.map(one, list(groups)):
            out[b, h * G:(h + 1) * G] = o
            lse[b, h * G:(h + 1) * G] = l
    return out, lse


def out_tolerance(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    with np.errstate(divide="ignore"):
        half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.maximum(a, 1e-300))) - 8), 0.0)
    return np.where(a < 4.0, OUT_TOL, half_ulp + 2e-3)


def assert_close(got, got_lse, ref, ref_lse, what=""):
    """Compare where the reference was computed (non-NaN).  Returns the max
    errors for reporting."""
    m = ~np.isnan(ref)
    assert m.any()
    assert np.all(np.isfinite(got[m])), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = out_tolerance(ref)
    bad = m & (err > tol)
    assert not bad.any(), (f"{what}: {int(bad.sum())} outputs beyond tolerance, "
                           f"max |dO| = {float(np.nanmax(np.where(m, err, np.nan))):.3e}")
    lm = ~np.isnan(ref_lse)
    empty = lm & np.isneginf(ref_lse)
    assert np.all(np.isneginf(got_lse[empty])), f"{what}: empty rows need lse = -inf"
    if empty.any():
        assert np.all(got[empty] == 0.0), f"{what}: empty rows need out = 0"
    fin = lm & ~empty
    lerr = np.abs(got_lse[fin] - ref_lse[fin]) if fin.any() else np.zeros(1)
    assert np.all(lerr <= LSE_TOL), f"{what}: max |dlse| = {float(lerr.max()):.3e}"
    return float(np.nanmax(np.where(m, err, np.nan))), float(lerr.max())


def big_outputs(ref) -> int:
    """Outputs whose magnitude puts bf16 rounding above 1e-2 (reported)."""
    return int(np.sum(np.abs(ref[~np.isnan(ref)]) >= 4.0))


def free_device():
    t = torch()
    import gc
    gc.collect()
    t.cuda.empty_cache()
