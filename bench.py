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
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        self.path = None
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

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.strip().split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"samples": 0}
        sm = [float(r[0]) for r in rows]
        mx = [float(r[1]) for r in rows]
        util = [float(r[3]) if r[3].replace(".", "").isdigit() else 0.0 for r in rows]
        loaded = [s for s, u in zip(sm, util) if u > 0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[2]) for r in rows)}


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

    def __init__(self, torch, fd, w, device, num_splits=None, copies=1):
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
                                    w.k_scale, w.v_scale)
        if num_splits:
            self.S = num_splits
        else:  # the planner over the whole problem, lengths included when known
            self.S = fd.fd_plan_problem(0, self.prob, w.seqlens)
        assert self.S >= 1, fd.fd_status_string(self.S)
        chunk = fd.fd_split_chunk(w.max_len, self.S)
        self.s_eff = max(1, -(-w.max_len // chunk)) if w.max_len else 1
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
    call = Call(torch, fd, w, device, args.splits, copies)

    sampler = ClockSampler(device.index)
    sampler.start()
    ms = timed(torch, call, args.steps, args.warmup, barrier)
    clocks = sampler.stop()
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
        "vs_baseline": None, "dtype": "bf16" if w.kv_dtype == "bf16" else "e4m3 cache, f16 mma",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "max_len": w.max_len, "block_size": w.block_size, "num_splits": call.S,
                   "effective_splits": call.s_eff, "kv_bytes_per_call": kvb,
                   "l2": f"inputs rotate over {copies} cache copies "
                         f"({copies * (w.k.nbytes + w.v.nbytes) / 1e6:.0f} MB, L2 {l2 / 1e6:.0f} MB)",
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        # achieved: algorithmic bytes over the whole call's event-timed duration
        # (the split kernel, the dominant one, plus the combine), so it is a
        # lower bound for the split kernel alone; traffic: the split kernel's
        # DRAM bytes per launch from ncu
        "roofline": {"bound": "hbm", "kernel": "fd_decode (split + combine)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4),
                     "traffic": ncu_traffic(w.name, call.S), "traffic_kernel": "fd_split_kernel",
                     "algorithmic_bytes": kvb},
        "gpu_launches": args.steps * call.launches_per_call,
        "clocks": clocks,
        "planner": planner_cost(fd, call.prob, w.seqlens),
    }

    if not args.no_e2e:
        result["e2e"] = e2e(torch, fd, call, w, device, min(args.steps, 30), 3, barrier, world)

    if not args.no_sweep and args.workload == "codellama34b" and rank == 0 and world == 1:
        result["sweep"] = sweep(torch, fd, device)

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


def sweep(torch, fd, device):
    from split_kv_decode_attn_b200 import workloads as wl
    peak, _ = measured_peak()
    rows = []
    for L in wl.CONFIG2_LENGTHS:
        w = wl.config(2, L=L)
        copies, _ = copies_for(torch, w.k.nbytes + w.v.nbytes, device)
        call = Call(torch, fd, w, device, None, copies)
        steps = max(200, min(20000, int(0.3e9 / max(w.kv_bytes(), 1) * 100)))
        ms = timed(torch, call, steps, 50)
        per = ms / 1e3 / steps
        gbs = w.kv_bytes() / per / 1e9
        g_us = timed_graph(torch, call, copies, max(1, steps // copies))
        g_gbs = w.kv_bytes() / (g_us * 1e-6) / 1e9
        rows.append({"L": L, "num_splits": call.S, "effective_splits": call.s_eff,
                     "us_per_call": round(per * 1e6, 3), "GB/s": round(gbs, 1),
                     "frac_measured": round(gbs / peak, 4), "frac_spec": round(gbs / SPEC_HBM_GBS, 4),
                     "graph_us_per_call": round(g_us, 3), "graph_GB/s": round(g_gbs, 1),
                     "graph_frac_measured": round(g_gbs / peak, 4),
                     "copies": copies, "steps": steps})
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
    partial (fd_decode_partial), the all-gather of the partial results and
    their merge (fd_combine).  value = the whole history's K+V bytes over the
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
    o = torch.empty((B, Hq, D), dtype=torch.float32, device=device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=device)
    o_all = torch.empty((world, B, Hq, D), dtype=torch.float32, device=device)
    l_all = torch.empty((world, B, Hq), dtype=torch.float32, device=device)
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
            dist.all_gather_into_tensor(o_all, o)
            dist.all_gather_into_tensor(l_all, lse)
        else:
            o_all[0].copy_(o)
            l_all[0].copy_(lse)
        st = fd.fd_combine(world, B, Hq, D, o_all, l_all, out, lse_out, stream)
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
    over L = 2K..64K, and at B = 64 and 256 over L = 512..8K, bf16 and fp8
    caches; G=4; the varlen, paged and peaked workloads.  One JSON line per shape on stdout, with the planner's pick
    (fd_plan_problem) and its regret against the fastest measured count."""
    import torch
    import split_kv_decode_attn_b200 as fd
    from split_kv_decode_attn_b200 import workloads as wl
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    fd.load_library()
    ladder = (1, 2, 3, 4, 6, 8, 12, 16, 20, 24, 28, 32, 40, 48, 64)

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
    for B, Ls in ((64, (512, 2048, 8192)), (256, (512, 2048, 4096))):
        for L in Ls:
            run(lambda B=B, L=L: wl.make_problem(B, 64, 8, 128, L, wl.CONFIG_SEED_BASE + 200 + B,
                                                 name=f"B{B}-L{L}"),
                [1, 2, 3, 4], f"bigbatch-B{B}-L{L}-bf16")
    for kvd in ("bf16", "fp8"):
        run(lambda kvd=kvd: make_workload("varlen", None, 0, kv_dtype=kvd), [1, 2, 3, 4, 6, 8],
            f"varlen-{kvd}")
    run(lambda: make_workload("paged", None, 0), [1, 2, 3, 4, 6, 8], "paged-bf16")
    run(lambda: make_workload("peaked", None, 0), [8, 12, 16, 20, 24, 32, 48, 64], "peaked-bf16")
    assert fd.fd_check_device_error() == 0


# ------------------------------------------------------- reference arm

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
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                   "max_len": w.max_len},
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
