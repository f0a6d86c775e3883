#!/usr/bin/env python
"""Benchmark of split-KV decode attention on B200.

One step is one fd_decode call (split kernel plus combine kernel) over one
batch: by default the CodeLlama-34B-shaped per-layer decode (B=1, Hq=64,
Hkv=8, D=128, bf16 cache of 65,536 tokens) with the planner's split count.
The timed region holds exactly --steps calls, bracketed by a barrier and a
device synchronisation, timed with CUDA events on the launching stream.
Cache copies rotate between steps so that L2 never serves K/V.

Reported (one JSON line from rank 0):
  value        KV-read GB/s summed over ranks (algorithmic K+V bytes / time)
  us_per_call  microseconds per fd_decode call
  roofline     achieved GB/s of the call against the measured HBM copy peak
  e2e          the same metric through the C ABI from pinned host buffers,
               host<->device copies inside the timed region
  cpu_baseline the fp64 oracle on this host's cores, on a bounded sample
  samples      the same call timed again as >= 10 samples of >= 20 calls
               (each long enough for the clock sampler to see it): median,
               min and max microseconds per call, and the SM clocks read
               inside those windows
  kernels      the split and combine kernels' shares of the call, from the
               committed ncu launch list, and the split kernel's own time and
               bandwidth derived from them
  workloads    the other benchmark shapes, each as the median of >= 10
               samples: the tiny MHA case at 1, 2, 4 and 8 splits, the varlen
               batch, the paged cache, the peaked 256K history and the fp8
               cache at 64K
  sweep        the same call at cache lengths 512 .. 64K
  planner      host microseconds per fd_plan_problem call (outside the timed
               region)

Multi-GPU (torchrun, one rank per GPU): every rank decodes its own batch
(independent sequences; the path needs no collective), weak scaling.

--impl reference times the fp64 CPU oracle instead (the slow reference of
what the method computes), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention µs/call and KV-read GB/s (fraction of B200 HBM roofline)"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0

WORKLOADS = {
    # name: (config index, cache length)
    "codellama34b": (2, 65536),
    "tiny": (1, None),
    "varlen": (3, None),
    "paged": (4, None),
    "peaked": (5, None),
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=500)
    ap.add_argument("--impl", choices=["fd", "reference"], default="fd")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="codellama34b")
    ap.add_argument("--L", type=int, default=None, help="cache length of the codellama34b workload")
    ap.add_argument("--splits", type=int, default=None, help="override the planner's split count")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="cache element type (fp8: e4m3 codes with per-tensor scales)")
    ap.add_argument("--fp8-mma", choices=["mma_sync", "tcgen05"], default="mma_sync",
                    help="tensor-core path of an fp8 cache (fd_problem.fp8_mma)")
    ap.add_argument("--layout", choices=["HND", "NHD"], default="HND",
                    help="cache dimension order (heads outside tokens, or tokens outside heads)")
    ap.add_argument("--shard-sequence", action="store_true",
                    help="sequence-parallel: the ranks split one history (strong scaling)")
    ap.add_argument("--sparse", action="store_true",
                    help="sparse decode (low-bit scan + top-delta) on a peaked 256K workload")
    ap.add_argument("--delta", type=float, default=8.0, help="top-delta threshold (nats)")
    ap.add_argument("--crossover", action="store_true",
                    help="planner sweep: split-count ladders over batch, length, element type")
    ap.add_argument("--crossover-filter", default=None,
                    help="with --crossover: only the shapes whose tag contains this text")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other benchmark shapes (the workloads array)")
    ap.add_argument("--samples", type=int, default=10,
                    help="timing samples per shape beside the declared region (at least 10 "
                         "are taken; 0 skips them, e.g. for a profiler run)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU time budget of the oracle baseline sample")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the device code (the kernels and their PTX helpers), with
    comments and blank lines left out so that documentation edits keep it."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "split_kv_decode_attn_b200", "csrc")
    for name in ("fd_kernels.cuh", "fd_ptx.cuh"):
        with open(os.path.join(csrc, name)) as f:
            code = [re.sub(r"//.*$", "", line).rstrip() for line in f]
        h.update(name.encode() + b"\0" + "\n".join(x for x in code if x).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, num_splits: int):
    """DRAM bytes (read + write) per launch of the split kernel, the dominant
    kernel, from the committed ncu summary, if it was taken on the current
    device code at the same split count; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        if j.get("source_hash") != kernel_source_hash():
            return None
        entry = j.get("workloads", {}).get(workload)
        if entry is None or int(entry["num_splits"]) != num_splits:
            return None
        return float(entry["split_kernel_bytes"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms, each
    sample with its time stamp, so that samples can be matched to timing
    windows of the host clock."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        self.path = None
        self.rows = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            gid = None
        self.gid = gid

    def start(self):
        if not self.gid:
            return
        fd_, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd_)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    @staticmethod
    def _parse(line):
        parts = [p.strip() for p in line.strip().split(",")]
        if len(parts) < 10:
            return None
        try:
            t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            util = float(parts[4]) if parts[4].replace(".", "").isdigit() else 0.0
            return {"t": t, "sm": float(parts[1]), "max": float(parts[2]),
                    "power": float(parts[3]), "util": util,
                    "reasons": [ClockSampler.REASONS[i] for i in range(4)
                                if parts[6 + i].lower() == "active"]}
        except ValueError:
            return None

    @staticmethod
    def summary(rows):
        if not rows:
            return {"samples": 0}
        loaded = [r["sm"] for r in rows if r["util"] > 0] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted({x for r in rows for x in r["reasons"]}),
                "samples": len(rows), "power_w_max": max(r["power"] for r in rows)}

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        with open(self.path) as f:
            self.rows = [r for r in map(self._parse, f) if r is not None]
        os.unlink(self.path)
        return self.summary(self.rows)

    def within(self, windows):
        """Summary of the samples taken inside the host-time windows [(t0, t1)]."""
        inside = [r for r in self.rows if any(t0 <= r["t"] <= t1 for t0, t1 in windows)]
        return self.summary(inside)


# ------------------------------------------------------------- our arm

def dev_bf16(torch, a, device):
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


def host_cache(torch, a):
    """Cache array as a host tensor of its storage type (bf16 bits or e4m3 codes)."""
    import numpy as np
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint8:
        return torch.from_numpy(a)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)


class Call:
    """Device buffers and a bound fd_decode call for one workload; `copies`
    rotating cache copies keep L2 from serving K/V."""

    def __init__(self, torch, fd, w, device, num_splits=None, copies=1, fp8_mma=0):
        self.torch, self.fd, self.w = torch, fd, w
        self.q = dev_bf16(torch, w.q, device)
        k = host_cache(torch, w.k).to(device)
        v = host_cache(torch, w.v).to(device)
        self.ks = [k] + [k.clone() for _ in range(copies - 1)]
        self.vs = [v] + [v.clone() for _ in range(copies - 1)]
        self.seqlens = None if w.seqlens is None else torch.from_numpy(w.seqlens).to(device)
        self.table = None if w.block_table is None else torch.from_numpy(w.block_table).to(device)
        self.prob = fd.make_problem(w.B, w.Hq, w.Hkv, w.D, w.max_len, w.block_size, w.num_blocks,
                                    w.max_blocks_per_seq, w.kv_layout, w.kv_dtype_code,
                                    w.k_scale, w.v_scale, fp8_mma)
        if num_splits:
            self.S = num_splits
        else:  # the planner over the whole problem, lengths included when known
            self.S = fd.fd_plan_problem(0, self.prob, w.seqlens)
        assert self.S >= 1, fd.fd_status_string(self.S)
        self.s_eff = fd.fd_effective_splits(w.max_len, self.S)
        self.out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=device)
        self.wbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.D, self.S)
        self.ws = torch.empty(max(self.wbytes, 4) // 4, dtype=torch.float32, device=device)
        self.stream = torch.cuda.current_stream(device).cuda_stream
        self.i = 0
        self.launches_per_call = 2 if self.s_eff > 1 else 1

    def __call__(self, k=None, v=None, q=None):
        c = self.i % len(self.ks)
        self.i += 1
        st = self.fd.fd_decode(self.prob, q if q is not None else self.q,
                               k if k is not None else self.ks[c], v if v is not None else self.vs[c],
                               self.seqlens, self.table, self.w.scale, self.S, self.out, self.lse,
                               self.ws, self.wbytes, self.stream)
        if st != 0:
            raise RuntimeError(f"fd_decode: {self.fd.fd_status_string(st)}")


def planner_cost(fd, prob, seqlens, num_sms=0, calls=2000):
    """Host microseconds per fd_plan_problem call through the Python binding,
    with the lengths when the workload has them (the planner runs outside the
    timed region; this is its cost).  None if the planner fails."""
    try:
        first = fd.fd_plan_problem(num_sms, prob, seqlens)
        if first < 1:
            return None
        t0 = time.perf_counter()
        for _ in range(calls):
            fd.fd_plan_problem(num_sms, prob, seqlens)
        dt = time.perf_counter() - t0
        return {"us_per_call": round(dt / calls * 1e6, 3), "calls": calls, "num_splits": first,
                "with_lengths": seqlens is not None}
    except Exception:
        return None


def max_over_ranks(torch, ms, world, device=None):
    """The slowest rank's time: the job is done when every rank is done."""
    if world <= 1:
        return float(ms)
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step, ms_total, steps, world):
    """Whole-job GB/s: every rank's algorithmic bytes over the slowest rank's time."""
    per_step_s = ms_total / 1e3 / steps
    return world * bytes_per_rank_step / per_step_s / 1e9


def timed(torch, fn, steps, warmup, barrier=None):
    for _ in range(warmup):
        fn()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return e0.elapsed_time(e1)  # ms


def sampled(torch, fn, samples, min_calls=20, min_window_s=0.25):
    """`samples` timing samples of back-to-back calls, each of at least
    `min_calls` calls and about `min_window_s` seconds (so that the 200 ms
    clock sampler sees every window), each timed with CUDA events on the
    launching stream with a device synchronisation on both sides.  Returns
    (microseconds per call of each sample, host-time windows, calls per
    sample)."""
    est = timed(torch, fn, min_calls, 3) * 1e3 / min_calls
    calls = max(min_calls, int(min_window_s * 1e6 / max(est, 1e-3)))
    per, windows = [], []
    for _ in range(max(samples, 1)):
        t0 = time.time()
        ms = timed(torch, fn, calls, 0)
        windows.append((t0, time.time()))
        per.append(ms * 1e3 / calls)
    return per, windows, calls


def sample_stats(per, calls, kv_bytes, peak):
    """Median, min and max of per-call samples, with bandwidth at the median
    against the measured copy peak and the 8 TB/s spec."""
    med = statistics.median(per)
    gbs = kv_bytes / med / 1e3
    return {"us_per_call_median": round(med, 3), "us_per_call_min": round(min(per), 3),
            "us_per_call_max": round(max(per), 3), "samples": len(per),
            "calls_per_sample": calls, "GB/s": round(gbs, 1),
            "frac_measured": round(gbs / peak, 4), "frac_spec": round(gbs / SPEC_HBM_GBS, 4)}


def workload_config(w, S, s_eff, copies, l2, world):
    """The `config` object of a bench line: the workload, the split count and
    how L2 is kept from serving K/V.  The reference arm reports the same."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "max_len": w.max_len, "block_size": w.block_size, "num_splits": S,
            "effective_splits": s_eff, "kv_bytes_per_call": w.kv_bytes(),
            "l2": f"inputs rotate over {copies} cache copies "
                  f"({copies * (w.k.nbytes + w.v.nbytes) / 1e6:.0f} MB, L2 {l2 / 1e6:.0f} MB)",
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def ncu_launch_shares(workload: str, num_splits: int):
    """Shares of the split and combine kernels in the committed ncu launch
    list (back-to-back calls, L2 not flushed between kernels), if it was
    taken on the current device code at the same split count; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        if j.get("source_hash") != kernel_source_hash():
            return None
        e = j.get("launches", {}).get(workload)
        if e is None or int(e["num_splits"]) != num_splits:
            return None
        return e
    except Exception:
        return None


def kernel_times(shares, us_per_call, kv_bytes, peak):
    """The split kernel's time inside the call, as its share of the launch
    list times the measured time per call, and its own bandwidth."""
    if not shares:
        return None
    split_us = shares["split_share"] * us_per_call
    return {"source": "ncu launch list (profiles/), shares x measured us/call",
            "split_share": shares["split_share"], "combine_share": shares["combine_share"],
            "split_ncu_us": shares["split_us"], "combine_ncu_us": shares["combine_us"],
            "split_us": round(split_us, 3), "split_GB/s": round(kv_bytes / split_us / 1e3, 1),
            "split_frac_measured": round(kv_bytes / split_us / 1e3 / peak, 4),
            "split_frac_spec": round(kv_bytes / split_us / 1e3 / SPEC_HBM_GBS, 4)}


# The other benchmark shapes of the default line: (workload, cache length,
# cache type, split counts; None = the planner's).
OTHER_WORKLOADS = (
    ("tiny", None, "bf16", (1, 2, 4, 8)),
    ("varlen", None, "bf16", (None,)),
    ("paged", None, "bf16", (None,)),
    ("peaked", None, "bf16", (None,)),
    ("codellama34b", 65536, "fp8", (None,)),
)


def other_workloads(torch, fd, device, n_samples):
    """Every other benchmark shape, each as the median of n_samples samples
    (plus the device time from CUDA-graph replays), with its split count,
    cache copies and the host-time windows of its samples (the caller turns
    them into the SM clocks seen inside them once the sampler has stopped)."""
    peak, _ = measured_peak()
    rows = []
    for name, L, kvd, splits in OTHER_WORKLOADS:
        w = make_workload(name, L, 0, kv_dtype=kvd)
        copies, l2 = copies_for(torch, w.k.nbytes + w.v.nbytes, device)
        for S in splits:
            call = Call(torch, fd, w, device, S, copies)
            per, windows, calls = sampled(torch, call, n_samples)
            g_us = timed_graph(torch, call, copies, max(1, 20 * calls // copies // 10))
            row = {"workload": w.name, "kv": kvd, "num_splits": call.S,
                   "effective_splits": call.s_eff, "kv_bytes_per_call": w.kv_bytes(),
                   "copies": copies}
            row.update(sample_stats(per, calls, w.kv_bytes(), peak))
            row["graph_us_per_call"] = round(g_us, 3)
            row["windows"] = windows     # replaced by the clocks seen inside them
            rows.append(row)
            del call
        del w
        torch.cuda.empty_cache()
    return rows


def timed_graph(torch, call, copies, reps, warmup=3):
    """Device time per call with the calls replayed from a CUDA graph (one
    captured call per cache copy): the cost of the call itself, free of the
    host's per-call launch work.  Returns microseconds per call."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    eager_stream = call.stream
    try:
        with torch.cuda.stream(s):
            call.stream = s.cuda_stream
            for _ in range(copies):
                call()  # one-time set-up happens outside the capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            call.stream = s.cuda_stream
            for _ in range(copies):
                call()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * copies) * 1e3
    finally:
        call.stream = eager_stream


def copies_for(torch, nbytes, device):
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    return max(2, math.ceil(4 * l2 / max(nbytes, 1))), l2


def make_workload(name, L, rank, nthreads=None, layout="HND", kv_dtype="bf16"):
    from split_kv_decode_attn_b200 import workloads as wl
    idx, default_L = WORKLOADS[name]
    if idx == 2:
        w = wl.config(2, L=L or default_L, nthreads=nthreads)
    else:
        w = wl.config(idx, nthreads=nthreads)
    if rank or layout != "HND" or kv_dtype != "bf16":
        # replicas: rank r decodes its own sequences (same shapes); the token-
        # major layout draws its cache in that storage order, fp8 caches
        # hold e4m3 codes
        suffix = ("" if layout == "HND" else "-NHD") + ("" if kv_dtype == "bf16" else "-fp8")
        w2 = wl.make_problem(w.B, w.Hq, w.Hkv, w.D, w.max_len, wl.CONFIG_SEED_BASE + 1000 * rank + idx,
                             seqlens=w.seqlens, nan_pad=w.seqlens is not None and not w.paged,
                             block_size=w.block_size, name=w.name + suffix,
                             nthreads=nthreads, layout=layout, kv_dtype=kv_dtype)
        if "dominant_positions" in w.meta and layout == "HND" and kv_dtype == "bf16":
            wl.plant_dominant_keys(w2, 64, wl.CONFIG_SEED_BASE + 1000 * rank + idx)
        w = w2
    return w


def oracle_sequence(w, b, off, n, threads):
    """The oracle on tokens [off, off + n) of sequence b, every query head.
    Returns the algorithmic K+V bytes of that window."""
    import numpy as np
    import oracle
    if w.kv_dtype == "fp8":  # dequantised cache: one fp64 oracle call per KV head
        from concurrent.futures import ThreadPoolExecutor
        from split_kv_decode_attn_b200 import workloads as wl
        G = w.G

        def head(h):
            k, v = w.logical_kv(b, h)
            k = float(np.float32(w.k_scale)) * wl.e4m3_bits_to_f64(k[off:off + n])
            v = float(np.float32(w.v_scale)) * wl.e4m3_bits_to_f64(v[off:off + n])
            oracle.attend_f64(wl.bf16_bits_to_f64(w.q[b, h * G:(h + 1) * G]), k, v,
                              float(np.float32(w.scale)))
        with ThreadPoolExecutor(max_workers=min(threads, w.Hkv)) as ex:
            list(ex.map(head, range(w.Hkv)))
        return n * w.Hkv * w.D * 2
    if w.paged or w.layout != "HND":
        kv = [w.logical_kv(b, h) for h in range(w.Hkv)]
        k = np.stack([x[0][off:off + n] for x in kv])[None]
        v = np.stack([x[1][off:off + n] for x in kv])[None]
    else:
        k, v = w.k[b:b + 1, :, off:off + n], w.v[b:b + 1, :, off:off + n]
    oracle.decode(w.q[b:b + 1], np.ascontiguousarray(k), np.ascontiguousarray(v), w.scale,
                  nthreads=threads)
    return n * w.Hkv * w.D * 4


def cpu_baseline(w, seconds):
    """The fp64 oracle, as it stands, on this host's cores: one sequence per
    oracle call (all its query heads, threads over heads), cycling through
    the batch until `seconds` of wall time have passed.  GB/s of algorithmic
    K+V bytes.  Then the same on one thread for a third of that time, over a
    window of each history sized to fit it."""
    cores = os.cpu_count() or 1
    threads = min(cores, w.Hq if w.kv_dtype == "bf16" else w.Hkv)
    lengths = w.lengths()

    def run(nthreads, limit, window):
        t0 = time.perf_counter()
        done = 0
        calls = 0
        while True:
            b = calls % w.B
            done += oracle_sequence(w, b, 0, min(window, int(lengths[b])), nthreads)
            calls += 1
            if time.perf_counter() - t0 >= limit:
                break
        return done, calls, time.perf_counter() - t0

    done, calls, dt = run(threads, seconds, int(lengths.max()))
    t1 = time.perf_counter()
    oracle_sequence(w, 0, 0, min(1024, int(lengths[0])), 1)
    per_tok = (time.perf_counter() - t1) / max(min(1024, int(lengths[0])), 1)
    window = int(max(64, min(int(lengths.max()), seconds / 3 / 4 / max(per_tok, 1e-9))))
    done1, calls1, dt1 = run(1, seconds / 3, window)
    return {"value": round(done / dt / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "hardware_threads": cores,
            "sample": f"{calls} oracle calls, each one whole sequence of the workload "
                      f"({w.Hq} query heads over its full history), {dt:.1f} s wall",
            "single_thread": {"value": round(done1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{calls1} oracle calls over the first {window} tokens "
                                        f"of a sequence, {dt1:.1f} s wall"}}


def run_fd(args):
    import torch
    import split_kv_decode_attn_b200 as fd

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
        barrier = lambda: dist.barrier(device_ids=[local])  # noqa: E731
    else:
        barrier = None
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    fd.load_library()

    w = make_workload(args.workload, args.L, rank, layout=args.layout, kv_dtype=args.kv_dtype)
    kvb = w.kv_bytes()
    copies, l2 = copies_for(torch, (w.k.nbytes + w.v.nbytes), device)
    tcgen05 = w.kv_dtype == "fp8" and args.fp8_mma == "tcgen05"
    call = Call(torch, fd, w, device, args.splits, copies,
                fd.FD_FP8_MMA_TCGEN05 if tcgen05 else fd.FD_FP8_MMA_SYNC)
    # ncu records are per kernel: the tcgen05 path has its own entries
    ncu_name = w.name + ("-tcgen05" if tcgen05 else "")

    sampler = ClockSampler(device.index)
    sampler.start()
    ms = timed(torch, call, args.steps, args.warmup, barrier)
    # Beside the declared region: the same call as >= 10 samples long enough
    # for the clock sampler (rank-local; reported by rank 0).
    n_samples = max(args.samples, 10) if args.samples > 0 else 0
    per, windows, calls = sampled(torch, call, n_samples) if n_samples else (None, None, None)
    workloads = None
    if n_samples and not args.no_workloads and rank == 0 and world == 1 \
            and args.workload == "codellama34b" and args.kv_dtype == "bf16" and args.layout == "HND":
        workloads = other_workloads(torch, fd, device, n_samples)
    clocks = sampler.stop()
    for row in workloads or ():
        row["clocks"] = sampler.within(row.pop("windows"))
    assert fd.fd_check_device_error() == 0

    ms = max_over_ranks(torch, ms, world, device)
    per_call_s = ms / 1e3 / args.steps
    value = job_throughput(kvb, ms, args.steps, world)
    peak, peak_kind = measured_peak()
    achieved = kvb / per_call_s / 1e9

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "us_per_call": round(per_call_s * 1e6, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.kv_dtype == "bf16" else
                 ("e4m3 cache, e4m3 tcgen05 mma" if tcgen05 else "e4m3 cache, f16 mma"),
        "data": "synthetic",
        "config": dict(workload_config(w, call.S, call.s_eff, copies, l2, world),
                       **({"fp8_mma": args.fp8_mma} if w.kv_dtype == "fp8" else {})),
        # achieved: algorithmic bytes over the whole call's event-timed duration
        # (the split kernel, the dominant one, plus the combine), so it is a
        # lower bound for the split kernel alone; traffic: the split kernel's
        # DRAM bytes per launch from ncu
        "roofline": {"bound": "hbm", "kernel": "fd_decode (split + combine)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4),
                     "traffic": ncu_traffic(ncu_name, call.S),
                     "traffic_kernel": "fd_split_tc_kernel" if tcgen05 else "fd_split_kernel",
                     "algorithmic_bytes": kvb},
        "gpu_launches": args.steps * call.launches_per_call,
        "clocks": clocks,
        "planner": planner_cost(fd, call.prob, w.seqlens),
    }
    if n_samples:
        stats = sample_stats(per, calls, kvb, peak)
        stats["clocks"] = sampler.within(windows)
        result["samples"] = stats
        result["kernels"] = kernel_times(ncu_launch_shares(ncu_name, call.S),
                                         stats["us_per_call_median"], kvb, peak)
    if workloads is not None:
        result["workloads"] = workloads

    if not args.no_e2e:
        result["e2e"] = e2e(torch, fd, call, w, device, min(args.steps, 30), 3, barrier, world)

    if not args.no_sweep and n_samples and args.workload == "codellama34b" and rank == 0 \
            and world == 1:
        result["sweep"] = sweep(torch, fd, device, n_samples)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)

    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def e2e(torch, fd, call, w, device, steps, warmup, barrier, world):
    """The same call from pinned host buffers: H2D of q, K, V, fd_decode,
    D2H of out and lse, all inside the timed region on one stream."""
    import numpy as np
    hq = torch.from_numpy(np.ascontiguousarray(w.q).view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = host_cache(torch, w.k).pin_memory()
    hv = host_cache(torch, w.v).pin_memory()
    dq, dk, dv = torch.empty_like(hq, device=device), torch.empty_like(hk, device=device), \
        torch.empty_like(hv, device=device)
    ho = torch.empty(call.out.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(call.lse.shape, dtype=torch.float32).pin_memory()

    def step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        call(dk, dv, dq)
        ho.copy_(call.out, non_blocking=True)
        hl.copy_(call.lse, non_blocking=True)

    ms = max_over_ranks(torch, timed(torch, step, steps, warmup, barrier), world, device)
    per = ms / 1e3 / steps
    h2d = hq.numel() * 2 + hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
    d2h = ho.numel() * 2 + hl.numel() * 4
    return {"value": round(job_throughput(w.kv_bytes(), ms, steps, world), 2), "unit": "GB/s",
            "us_per_call": round(per * 1e6, 1), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps}


def sweep(torch, fd, device, n_samples=10):
    from split_kv_decode_attn_b200 import workloads as wl
    peak, _ = measured_peak()
    rows = []
    for L in wl.CONFIG2_LENGTHS:
        w = wl.config(2, L=L)
        copies, _ = copies_for(torch, w.k.nbytes + w.v.nbytes, device)
        call = Call(torch, fd, w, device, None, copies)
        per, _, calls = sampled(torch, call, n_samples)
        g_us = timed_graph(torch, call, copies, max(1, 2 * calls // copies))
        g_gbs = w.kv_bytes() / (g_us * 1e-6) / 1e9
        row = {"L": L, "num_splits": call.S, "effective_splits": call.s_eff, "copies": copies}
        row.update(sample_stats(per, calls, w.kv_bytes(), peak))
        row.update({"graph_us_per_call": round(g_us, 3), "graph_GB/s": round(g_gbs, 1),
                    "graph_frac_measured": round(g_gbs / peak, 4)})
        kt = kernel_times(ncu_launch_shares(w.name, call.S), row["us_per_call_median"],
                          w.kv_bytes(), peak)
        if kt:
            row["kernels"] = kt
        rows.append(row)
        del call
        torch.cuda.empty_cache()
    return rows


def run_sparse(args):
    """fd_decode_sparse against fd_decode on the peaked 256K shape (B=1, Hq=32,
    Hkv=8, D=128).  Workload "peaked" (the default workload name maps here to
    the group-peaked keys, which dominate every head of a group) or the
    benchmark's own peaked workload (--workload peaked: keys that dominate one
    head per group).  The key codes are made once, outside the timed region
    (in a decode loop they change only where tokens are appended).  Reports
    the sparse call's time, the bytes it must read (codes of every token plus
    K and V of the kept blocks) against the HBM peak, the dense call's time
    and the speed-up."""
    import numpy as np
    import torch
    import split_kv_decode_attn_b200 as fd
    from split_kv_decode_attn_b200 import workloads as wl
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    fd.load_library()
    w = wl.config(5) if args.workload == "peaked" else wl.peaked_group()
    copies = 2
    call = Call(torch, fd, w, device, None, copies)
    S = call.S
    nblk = -(-w.max_len // 64)
    k8s, sks = [], []
    for c in range(copies):
        k8 = torch.empty(w.k.shape, dtype=torch.int8, device=device)
        sk = torch.empty((w.B, w.Hkv, nblk), dtype=torch.float32, device=device)
        assert fd.fd_quantize_keys(call.prob, call.ks[c], call.seqlens, k8, sk) == 0
        k8s.append(k8)
        sks.append(sk)
    kept = torch.empty((w.B, w.Hkv, nblk), dtype=torch.uint8, device=device)
    out_s = torch.empty_like(call.out)
    lse_s = torch.empty_like(call.lse)
    state = {"i": 0}

    def sparse_call():
        c = state["i"] % copies
        state["i"] += 1
        st = fd.fd_decode_sparse(call.prob, call.q, call.ks[c], call.vs[c], k8s[c], sks[c],
                                 call.seqlens, w.scale, args.delta, S, out_s, lse_s, kept,
                                 call.ws, call.wbytes, call.stream)
        if st != 0:
            raise RuntimeError(f"fd_decode_sparse: {fd.fd_status_string(st)}")

    steps, warmup = args.steps, args.warmup
    sampler = ClockSampler(device.index)
    sampler.start()
    ms_sparse = timed(torch, sparse_call, steps, warmup)
    clocks = sampler.stop()
    ms_dense = timed(torch, call, steps, warmup)
    us_sparse = ms_sparse * 1e3 / steps
    us_dense = ms_dense * 1e3 / steps
    # one more call of each on the same copy, for the kept share and the gap
    state["i"] = 0
    sparse_call()
    call.i = 0
    call()
    torch.cuda.synchronize()
    assert fd.fd_check_device_error() == 0
    kept_np = kept.cpu().numpy().astype(bool)
    share = float(kept_np.mean())
    gap = float((out_s.float() - call.out.float()).abs().max())
    lse_gap = float((lse_s - call.lse).abs().max())
    n_tok = int(w.lengths().sum())
    read = n_tok * w.Hkv * w.D + int(kept_np.sum()) * 64 * w.D * 4   # codes + kept K, V
    dense_bytes = w.kv_bytes()
    peak, peak_kind = measured_peak()
    achieved = read / (us_sparse * 1e-6) / 1e9
    print(json.dumps({
        "metric": "sparse decode µs/call and bytes-read GB/s (fraction of B200 HBM roofline)",
        "value": round(achieved, 1), "unit": "GB/s", "n_gpus": 1, "steps": steps,
        "warmup": warmup, "us_per_call": round(us_sparse, 3), "higher_is_better": True,
        "dtype": "bf16 attention, int8 scan", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "max_len": w.max_len, "num_splits": S, "delta": args.delta,
                   "l2": f"inputs rotate over {copies} copies of K, V and the codes"},
        "kept_block_share": round(share, 5),
        "bytes_read_per_call": read, "dense_kv_bytes_per_call": dense_bytes,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": ncu_traffic(w.name, S) if args.delta == 8.0 else None,
                     "traffic_kernel": "fd_split_kernel (sparse)"},
        "dense": {"us_per_call": round(us_dense, 3),
                  "GB/s": round(dense_bytes / (us_dense * 1e-6) / 1e9, 1)},
        "speedup_vs_dense": round(us_dense / us_sparse, 3),
        "dense_equivalent_GB/s": round(dense_bytes / (us_sparse * 1e-6) / 1e9, 1),
        "vs_dense_max_abs_dout": gap, "vs_dense_max_abs_dlse": lse_gap,
        "gpu_launches": steps * call.launches_per_call,
        "clocks": clocks,
    }), flush=True)


def run_sharded(args):
    """Sequence-parallel decode of the CodeLlama-34B-shaped workload: rank r
    holds tokens [r*L/N, (r+1)*L/N) of every KV head.  A step is the local
    partial (fd_decode_partial) written into one packed buffer, one
    all-gather of the packed buffers and their merge where they lie
    (fd_combine_strided).  value = the whole history's K+V bytes over the
    slowest rank's time (strong scaling)."""
    import numpy as np
    import torch
    import split_kv_decode_attn_b200 as fd
    from split_kv_decode_attn_b200 import sharded
    from split_kv_decode_attn_b200 import workloads as wl

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
        barrier = lambda: dist.barrier(device_ids=[local])  # noqa: E731
    else:
        barrier = None
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    fd.load_library()
    L = args.L or WORKLOADS["codellama34b"][1]
    w = wl.config(2, L=L)  # every rank draws the same history and keeps its slice
    lo, hi = sharded.shard_bounds(L, world, rank)
    q = dev_bf16(torch, w.q, device)
    k0 = dev_bf16(torch, np.ascontiguousarray(w.k[:, :, lo:hi]), device)
    v0 = dev_bf16(torch, np.ascontiguousarray(w.v[:, :, lo:hi]), device)
    copies, _ = copies_for(torch, k0.numel() * 4, device)  # rotate slices past L2
    ks = [k0] + [k0.clone() for _ in range(copies - 1)]
    vs = [v0] + [v0.clone() for _ in range(copies - 1)]
    turn = [0]
    B, Hq, D, Hkv = w.B, w.Hq, w.D, w.Hkv
    prob = fd.make_problem(B, Hq, Hkv, D, hi - lo)
    S = args.splits or fd.fd_plan(B, Hq, Hkv, D, hi - lo, 0)
    nbytes = fd.fd_workspace_bytes(B, Hq, D, S)
    ws = torch.empty(max(nbytes, 4) // 4, dtype=torch.float32, device=device)
    # This rank's partial goes straight into its packed buffer (O rows, then
    # lse); one all-gather lays the ranks' buffers end to end, and the merge
    # reads them where they lie.  With one rank the packed buffer is the
    # gathered one.
    P = sharded.packed_floats(B, Hq, D)
    send = torch.empty(P, dtype=torch.float32, device=device)
    parts = torch.empty(world * P, dtype=torch.float32, device=device) if world > 1 else send
    o, lse = sharded.unpack(send, B, Hq, D)
    rows = B * Hq
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=device)
    lse_out = torch.empty((B, Hq), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device).cuda_stream

    def step():
        c = turn[0] % copies
        turn[0] += 1
        st = fd.fd_decode_partial(prob, q, ks[c], vs[c], None, None, w.scale, S, o, lse, ws,
                                  nbytes, stream)
        assert st == 0, fd.fd_status_string(st)
        if world > 1:
            import torch.distributed as dist
            dist.all_gather_into_tensor(parts, send)
        base = parts.data_ptr()
        st = fd.fd_combine_strided(world, B, Hq, D, base, P, base + 4 * rows * D, P, out,
                                   lse_out, stream)
        assert st == 0, fd.fd_status_string(st)

    ms = max_over_ranks(torch, timed(torch, step, args.steps, args.warmup, barrier), world, device)
    assert fd.fd_check_device_error() == 0
    kvb = w.kv_bytes()
    per = ms / 1e3 / args.steps
    peak, peak_kind = measured_peak()
    result = {
        "metric": METRIC, "value": round(kvb / per / 1e9, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "us_per_call": round(per * 1e6, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name + f"-seq{world}", "B": B, "Hq": Hq, "Hkv": Hkv, "D": D,
                   "max_len": L, "tokens_per_rank": hi - lo, "num_splits": S,
                   "l2": f"each rank rotates {copies} copies of its slice",
                   "parallelism": f"seq{world}"},
        "roofline": {"bound": "hbm", "achieved": round(kvb / world / per / 1e9, 1),
                     "peak": peak, "unit": "GB/s", "peak_kind": peak_kind,
                     "frac": round(kvb / world / per / 1e9 / peak, 4), "traffic": None},
        "gpu_launches": args.steps * ((2 if S > 1 else 1) + 1),
    }
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def crossover(args):
    """Split-count sweep for the planner: device microseconds per fd_decode
    call over a ladder of split counts, timed from CUDA-graph replays (the
    call's own cost; eager calls below ~2K tokens are bound by the host's
    launch work), with cache copies rotated past L2.  Shapes: the CodeLlama-34B
    head shape (Hq=64, Hkv=8, D=128) at B=1 over L = 512..128K, at B = 2..40
    over L = 2K..64K, and at B = 64 and 256 over L = 512..64K and 512..16K, bf16 and fp8
    caches; G=4; the varlen, paged and peaked workloads.  One JSON line per shape on stdout, with the planner's pick
    (fd_plan_problem) and its regret against the fastest measured count."""
    import torch
    import split_kv_decode_attn_b200 as fd
    from split_kv_decode_attn_b200 import workloads as wl
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    fd.load_library()
    ladder = (1, 2, 3, 4, 6, 8, 12, 16, 18, 20, 24, 28, 32, 40, 48, 64)

    def run(make, Ss, tag):
        """make: builds the workload (only for the shapes that are run)."""
        if args.crossover_filter and args.crossover_filter not in tag:
            return
        w = make()
        copies, _ = copies_for(torch, w.k.nbytes + w.v.nbytes, device)
        prob = fd.make_problem(w.B, w.Hq, w.Hkv, w.D, w.max_len, w.block_size, w.num_blocks,
                               w.max_blocks_per_seq, w.kv_layout, w.kv_dtype_code, w.k_scale,
                               w.v_scale)
        plan = fd.fd_plan_problem(0, prob, w.seqlens)
        times = {}
        for S in sorted(set(Ss) | {plan}):
            call = Call(torch, fd, w, device, S, copies)
            est = timed_graph(torch, call, copies, 3, warmup=1)
            times[S] = timed_graph(torch, call, copies, max(3, int(60000 / max(est, 1.0) / copies)))
            del call
        torch.cuda.empty_cache()
        best = min(times, key=times.get)
        kv = w.kv_bytes()
        print(json.dumps({"tag": tag, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "L": w.max_len,
                          "bs": w.block_size, "kv": w.kv_dtype, "kv_bytes": kv, "plan": plan,
                          "us": {str(k): round(v, 2) for k, v in sorted(times.items())},
                          "best": best, "plan_regret": round(times[plan] / times[best] - 1, 4),
                          "plan_GBs": round(kv / times[plan] / 1e3, 1)}), flush=True)

    for L in (512, 1024, 2048, 4096, 8192, 16384, 32768, 65536, 131072):
        for kvd in ("bf16", "fp8"):
            run(lambda L=L, kvd=kvd: make_workload("codellama34b", L, 0, kv_dtype=kvd),
                [s for s in ladder if s <= L // 64], f"B1-L{L}-{kvd}")
    for L in (16384, 65536):
        run(lambda L=L: wl.make_problem(1, 32, 8, 128, L, wl.CONFIG_SEED_BASE + 300, name="g4"),
            [s for s in ladder if s <= L // 64], f"G4-B1-L{L}")
    for B in (2, 4, 8, 16, 32, 40):
        for L in (2048, 8192, 16384, 65536):
            if B * 8 * L * 128 * 4 > 4.5e9:
                continue
            for kvd in (("bf16", "fp8") if B in (4, 16) else ("bf16",)):
                run(lambda B=B, L=L, kvd=kvd: wl.make_problem(
                        B, 64, 8, 128, L, wl.CONFIG_SEED_BASE + 200 + B, name=f"B{B}-L{L}",
                        kv_dtype=kvd),
                    [s for s in (1, 2, 3, 4, 6, 8, 12, 16, 24, 32) if s <= L // 64],
                    f"B{B}-L{L}-{kvd}")
    # Large batches: B * Hkv = 512 and 2048 CTAs at S = 1 already fill the device.
    # Up to 64K tokens at B = 64 and 16K at B = 256 (17 GB of cache each).
    for B, Ls in ((64, (512, 2048, 8192, 16384, 32768, 65536)),
                  (256, (512, 2048, 4096, 16384))):
        for L in Ls:
            run(lambda B=B, L=L: wl.make_problem(B, 64, 8, 128, L, wl.CONFIG_SEED_BASE + 200 + B,
                                                 name=f"B{B}-L{L}"),
                [1, 2, 3, 4], f"bigbatch-B{B}-L{L}-bf16")
    for kvd in ("bf16", "fp8"):
        run(lambda kvd=kvd: make_workload("varlen", None, 0, kv_dtype=kvd), [1, 2, 3, 4, 6, 8],
            f"varlen-{kvd}")
    run(lambda: make_workload("paged", None, 0), [1, 2, 3, 4, 6, 8], "paged-bf16")
    run(lambda: make_workload("paged", None, 0, kv_dtype="fp8"), [2, 3, 4, 6, 8, 9, 12],
        "paged-fp8")
    run(lambda: make_workload("peaked", None, 0), [8, 12, 16, 20, 24, 32, 48, 64], "peaked-bf16")
    run(lambda: make_workload("peaked", None, 0, kv_dtype="fp8"), [16, 18, 24, 32, 48],
        "peaked-fp8")
    assert fd.fd_check_device_error() == 0


# ------------------------------------------------------- reference arm

def reference_config(w, world):
    """The repo arm's `config` for the same workload, so that the two lines
    name the same problem: the split count is what the planner (host code)
    picks for it, and the cache copies are those the repo arm rotates.  The
    oracle itself neither splits nor rotates anything."""
    import torch
    import split_kv_decode_attn_b200 as fd
    sms, l2 = 148, 126 * 1024 * 1024
    if torch.cuda.is_available():
        props = torch.cuda.get_device_properties(0)
        sms, l2 = props.multi_processor_count, props.L2_cache_size
    prob = fd.make_problem(w.B, w.Hq, w.Hkv, w.D, w.max_len, w.block_size, w.num_blocks,
                           w.max_blocks_per_seq, w.kv_layout, w.kv_dtype_code, w.k_scale,
                           w.v_scale)
    S = fd.fd_plan_problem(sms, prob, w.seqlens)
    copies = max(2, math.ceil(4 * l2 / max(w.k.nbytes + w.v.nbytes, 1)))
    return workload_config(w, S, fd.fd_effective_splits(w.max_len, S), copies, l2, world)


def run_reference(args):
    """The fp64 CPU oracle timed as the reference arm, on this host's cores.
    Each step is one bounded sample of the workload: every query head of one
    sequence (threads over heads) over a window of its history.  The window
    is calibrated so that the whole --steps/--warmup run takes about two
    minutes.  Rank 0 alone runs it."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = make_workload(args.workload, args.L, 0, layout=args.layout, kv_dtype=args.kv_dtype)
    cores = os.cpu_count() or 1
    threads = min(cores, w.Hq if w.kv_dtype == "bf16" else w.Hkv)
    lengths = w.lengths()
    seqs = [b for b in range(w.B) if lengths[b] > 0]
    budget_per_step = 120.0 / max(args.steps + args.warmup, 1)

    def sample(i, n_tok):
        b = seqs[i % len(seqs)]
        n = min(n_tok, int(lengths[b]))
        off = (i * 7919) % max(int(lengths[b]) - n + 1, 1)
        return oracle_sequence(w, b, off, n, threads)

    n_tok = 1024
    t0 = time.perf_counter()
    sample(0, n_tok)
    dt = max(time.perf_counter() - t0, 1e-6)
    n_tok = int(max(16, min(int(lengths.max()), n_tok * budget_per_step / dt)))
    for i in range(args.warmup):
        sample(i, n_tok)
    t0 = time.perf_counter()
    nbytes = 0
    for i in range(args.steps):
        nbytes += sample(i, n_tok)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": reference_config(w, world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: all {w.Hq} query heads of one sequence over a "
                                   f"{n_tok}-token window of its history, {threads} threads"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.crossover:
        crossover(args)
    elif args.shard_sequence:
        run_sharded(args)
    elif args.sparse:
        run_sparse(args)
    else:
        run_fd(args)


if __name__ == "__main__":
    main()
