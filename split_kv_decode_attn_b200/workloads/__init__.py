"""Seeded synthetic inputs for split-KV decode attention.

This module draws inputs only; it holds none of the attention arithmetic.
The test harness, the benchmark and the fp64 oracle all take their inputs
from here, so both sides of a parity check see the same bf16 bytes.

Every tensor element is a pure function of (stream seed, element index):
the SplitMix64 counter generator of ``fdgen.c`` followed by Box-Muller and
round-to-nearest-even to bf16.  bf16 tensors are held as ``numpy.uint16``
bit patterns.

Workload shapes follow the decode workload the Flash-Decoding write-up
discusses (one query token per sequence against a long cached history,
CodeLlama-34B at batch 1 over 512 to 64K tokens: slavadubrov.com, "What is
Flash-Decoding, and when does it speed up LLMs?", sections "Why decode needs
a different schedule" and "Interpret the reported result") plus the 256K
context of "Faster Than Flash" (abstract).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC_PATH = os.path.join(_HERE, "fdgen.c")
_LIB_PATH = os.path.join(_HERE, "libfdgen.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile fdgen.c into libfdgen.so next to it."""
    if (force or not os.path.exists(_LIB_PATH)
            or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC_PATH)):
        subprocess.check_call(["gcc", "-O2", "-Wall", "-Wextra", "-shared", "-fPIC",
                               "-pthread", _SRC_PATH, "-o", _LIB_PATH, "-lm"])
    return _LIB_PATH

BF16_NAN = np.uint16(0x7FC0)

# Stream indices: each tensor of a workload draws from its own stream, whose
# seed is draw number <index> of the workload's base stream.
STREAM_Q, STREAM_K, STREAM_V, STREAM_SEQLENS, STREAM_PERM, STREAM_POS = range(6)


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64 = ctypes.c_uint64
        lib.fdgen_u64.argtypes = [u64, u64, u64, ctypes.c_void_p]
        lib.fdgen_u64.restype = None
        lib.fdgen_normal_f64.argtypes = [u64, u64, u64, ctypes.c_void_p]
        lib.fdgen_normal_f64.restype = None
        lib.fdgen_normal_bf16.argtypes = [u64, u64, u64, ctypes.c_void_p, ctypes.c_int]
        lib.fdgen_normal_bf16.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def u64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    if n:
        _load().fdgen_u64(seed, offset, n, out.ctypes.data)
    return out


def normal_f64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    if n:
        _load().fdgen_normal_f64(seed, offset, n, out.ctypes.data)
    return out


def normal_bf16(seed: int, shape, offset: int = 0, out: Optional[np.ndarray] = None,
                nthreads: Optional[int] = None) -> np.ndarray:
    """bf16 bit patterns of N(0,1) draws, element i = draw (offset + i)."""
    n = int(np.prod(shape)) if len(shape) else 1
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    if n:
        _load().fdgen_normal_bf16(seed, offset, n, out.ctypes.data,
                                  nthreads or default_threads())
    return out


def stream_seed(base_seed: int, stream: int) -> int:
    return int(u64(base_seed, 1, offset=stream)[0])


def uniform_int(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers in [lo, hi]: lo + (draw mod (hi - lo + 1))."""
    r = u64(seed, n)
    return (np.int64(lo) + (r % np.uint64(hi - lo + 1)).astype(np.int64)).astype(np.int32)


def permutation(seed: int, n: int) -> np.ndarray:
    """Fisher-Yates: for i = n-1 .. 1, swap a[i] with a[draw_k mod (i+1)], k = n-1-i."""
    a = np.arange(n, dtype=np.int64)
    r = u64(seed, max(n - 1, 0))
    for k, i in enumerate(range(n - 1, 0, -1)):
        j = int(r[k] % np.uint64(i + 1))
        a[i], a[j] = a[j], a[i]
    return a.astype(np.int32)


def distinct_positions(seed: int, count: int, n: int) -> np.ndarray:
    """`count` distinct integers of [0, n): the first `count` steps of a
    forward Fisher-Yates shuffle of 0..n-1 (swap a[i] with a[i + draw_i mod (n-i)])."""
    r = u64(seed, count)
    swapped: dict = {}
    out = []
    for i in range(count):
        j = i + int(r[i] % np.uint64(n - i))
        ai, aj = swapped.get(i, i), swapped.get(j, j)
        swapped[i], swapped[j] = aj, ai
        out.append(aj)
    return np.array(out, dtype=np.int32)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (nearest even) -> bf16 (nearest even), as bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# OCP 8-bit floating point, E4M3: sign, 4 exponent bits (bias 7), 3 mantissa
# bits; exponent field 0 holds subnormals (m * 2^-9); S.1111.111 is NaN and
# there is no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.
E4M3_MAX = 448.0


def e4m3_bits_to_f64(c: np.ndarray) -> np.ndarray:
    c = np.asarray(c, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def f64_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round to nearest, ties to even, saturating at +-448 (finite input)."""
    x = np.asarray(x, dtype=np.float64)
    sign = (np.signbit(x)).astype(np.int64) << 7
    a = np.minimum(np.abs(x), E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)                      # binade; -6 also covers subnormals
    step = np.exp2(e - 3)
    q = np.rint(a / step) * step               # np.rint: ties to even
    q = np.minimum(q, E4M3_MAX)
    with np.errstate(divide="ignore"):
        qe = np.floor(np.log2(np.where(q > 0, q, 1.0)))
    normal = q >= 2.0 ** -6
    ef = np.where(normal, qe + 7, 0).astype(np.int64)
    mf = np.where(normal, q / np.exp2(qe) * 8 - 8, q / 2.0 ** -9)
    code = sign | (ef << 3) | np.rint(mf).astype(np.int64)
    return code.astype(np.uint8)


@dataclass
class Workload:
    """One decode-attention problem held on the host.

    q: [B, Hq, D] bf16 bits.  Cache layout "HND": contiguous k, v
    [B, Hkv, max_len, D], paged [num_blocks, Hkv, block_size, D].  Layout
    "NHD": contiguous [B, max_len, Hkv, D], paged [num_blocks, block_size,
    Hkv, D].  Paged caches come with block_table [B, max_blocks_per_seq]
    int32.  seqlens: [B] int32 or None (every sequence holds max_len)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    max_len: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    scale: float
    seqlens: Optional[np.ndarray] = None
    block_size: int = 0
    block_table: Optional[np.ndarray] = None
    layout: str = "HND"
    kv_dtype: str = "bf16"         # "bf16" (uint16 bits) or "fp8" (e4m3 codes, uint8)
    k_scale: float = 1.0           # fp8: real K = k_scale * code
    v_scale: float = 1.0
    meta: dict = field(default_factory=dict)

    @property
    def kv_dtype_code(self) -> int:
        return 0 if self.kv_dtype == "bf16" else 1

    @property
    def kv_layout(self) -> int:
        return 0 if self.layout == "HND" else 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    @property
    def num_blocks(self) -> int:
        return int(self.k.shape[0]) if self.paged else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1]) if self.paged else 0

    def lengths(self) -> np.ndarray:
        if self.seqlens is None:
            return np.full(self.B, self.max_len, dtype=np.int64)
        return np.clip(self.seqlens.astype(np.int64), 0, self.max_len)

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes: valid tokens x Hkv x D x element bytes x 2."""
        elem = 2 if self.kv_dtype == "bf16" else 1
        return int(self.lengths().sum()) * self.Hkv * self.D * elem * 2

    def logical_kv_f64(self, b: int, h: int):
        """Real (dequantised) K, V rows [n, D] of sequence b, KV head h, in fp64."""
        k, v = self.logical_kv(b, h)
        if self.kv_dtype == "bf16":
            return bf16_bits_to_f64(k), bf16_bits_to_f64(v)
        return (float(np.float32(self.k_scale)) * e4m3_bits_to_f64(k),
                float(np.float32(self.v_scale)) * e4m3_bits_to_f64(v))

    def logical_kv(self, b: int, h: int):
        """K, V rows [n, D] (bf16 bits) of sequence b, KV head h, in token order."""
        n = int(self.lengths()[b])
        hnd = self.layout == "HND"
        if not self.paged:
            if hnd:
                return self.k[b, h, :n], self.v[b, h, :n]
            return self.k[b, :n, h], self.v[b, :n, h]
        bs = self.block_size
        npages = (n + bs - 1) // bs
        pages = self.block_table[b, :npages].astype(np.int64)
        if hnd:
            kk, vv = self.k[pages, h], self.v[pages, h]
        else:
            kk, vv = self.k[pages, :, h], self.v[pages, :, h]
        return kk.reshape(-1, self.D)[:n], vv.reshape(-1, self.D)[:n]


def make_problem(B: int, Hq: int, Hkv: int, D: int, max_len: int, seed: int,
                 seqlens=None, nan_pad: bool = False, block_size: int = 0,
                 num_blocks: Optional[int] = None, name: str = "custom",
                 nthreads: Optional[int] = None, layout: str = "HND", kv_dtype: str = "bf16",
                 kv_scale: float = 1.0 / 32) -> Workload:
    """Build a workload with i.i.d. N(0,1) bf16 q, K, V from base `seed`.

    Contiguous cache when block_size == 0.  Paged cache otherwise: the
    physical pool holds `num_blocks` pages (default: exactly enough for every
    sequence) and the block table is a seeded permutation of the pool,
    reshaped [B, max_len / block_size].  `layout` orders the cache dims
    ("HND": heads outside tokens, "NHD": tokens outside heads); K and V are
    drawn in the storage order of that layout.  kv_dtype "fp8": K and V hold
    e4m3 codes of N(0,1) / kv_scale (so the real values, kv_scale * code, are
    N(0,1) rounded to e4m3), with k_scale = v_scale = kv_scale."""
    assert layout in ("HND", "NHD") and kv_dtype in ("bf16", "fp8")
    q = normal_bf16(stream_seed(seed, STREAM_Q), (B, Hq, D), nthreads=nthreads)
    if block_size:
        assert max_len % block_size == 0
        per_seq = max_len // block_size
        nb = num_blocks if num_blocks is not None else B * per_seq
        assert nb >= B * per_seq
        perm = permutation(stream_seed(seed, STREAM_PERM), nb)
        table = perm[: B * per_seq].reshape(B, per_seq).copy()
        shape = (nb, Hkv, block_size, D) if layout == "HND" else (nb, block_size, Hkv, D)
    else:
        table = None
        shape = (B, Hkv, max_len, D) if layout == "HND" else (B, max_len, Hkv, D)
    if kv_dtype == "bf16":
        k = normal_bf16(stream_seed(seed, STREAM_K), shape, nthreads=nthreads)
        v = normal_bf16(stream_seed(seed, STREAM_V), shape, nthreads=nthreads)
    else:
        n = int(np.prod(shape))
        k = f64_to_e4m3_bits(normal_f64(stream_seed(seed, STREAM_K), n) / kv_scale).reshape(shape)
        v = f64_to_e4m3_bits(normal_f64(stream_seed(seed, STREAM_V), n) / kv_scale).reshape(shape)
    sl = None if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    if nan_pad and sl is not None:
        assert not block_size
        nan = BF16_NAN if kv_dtype == "bf16" else np.uint8(0x7F)
        for b in range(B):
            if layout == "HND":
                k[b, :, int(sl[b]):, :] = nan
                v[b, :, int(sl[b]):, :] = nan
            else:
                k[b, int(sl[b]):, :, :] = nan
                v[b, int(sl[b]):, :, :] = nan
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, max_len=max_len, q=q, k=k, v=v,
                    scale=float(np.float32(1.0 / math.sqrt(D))), seqlens=sl,
                    block_size=block_size, block_table=table, layout=layout, kv_dtype=kv_dtype,
                    k_scale=kv_scale if kv_dtype == "fp8" else 1.0,
                    v_scale=kv_scale if kv_dtype == "fp8" else 1.0)


def plant_dominant_keys(w: Workload, count: int, seed: int, magnitude: float = 4.0) -> np.ndarray:
    """Overwrite `count` seeded distinct positions of every KV head with the key
    magnitude * q/|q| * sqrt(D), q being the group's first query head of that
    KV head (batch entry 0 .. B-1 alike), computed in fp64 and rounded to bf16.
    Returns the positions."""
    assert not w.paged and w.layout == "HND"
    pos = distinct_positions(stream_seed(seed, STREAM_POS), count, w.max_len)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            q0 = bf16_bits_to_f64(w.q[b, h * G])
            key = magnitude * q0 / np.linalg.norm(q0) * math.sqrt(w.D)
            w.k[b, h, pos, :] = f64_to_bf16_bits(key)[None, :]
    w.meta["dominant_positions"] = pos
    return pos


def plant_group_keys(w: Workload, count: int, seed: int, magnitude: float = 4.0) -> np.ndarray:
    """Like plant_dominant_keys, but the key follows the normalised sum of all
    query heads of the group, magnitude * u * sqrt(D) with u = sum_g q_g /
    |sum_g q_g|, so that it stands out for every head of the group (the
    sparse decode's peaked input).  Returns the positions."""
    assert not w.paged and w.layout == "HND"
    pos = distinct_positions(stream_seed(seed, STREAM_POS), count, w.max_len)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            u = bf16_bits_to_f64(w.q[b, h * G:(h + 1) * G]).sum(axis=0)
            key = magnitude * u / np.linalg.norm(u) * math.sqrt(w.D)
            w.k[b, h, pos, :] = f64_to_bf16_bits(key)[None, :]
    w.meta["dominant_positions"] = pos
    return pos


def peaked_group(nthreads: Optional[int] = None) -> Workload:
    """The peaked workload's shape (B=1, Hq=32, Hkv=8, D=128, L=262144) with its
    64 dominant keys aligned with the whole query group (plant_group_keys)."""
    seed = CONFIG_SEED_BASE + 6
    w = make_problem(1, 32, 8, 128, 262144, seed, name="peaked-group-L256K", nthreads=nthreads)
    plant_group_keys(w, 64, seed)
    return w


# --- the five workloads -------------------------------------------------------

CONFIG_SEED_BASE = 20260000
CONFIG2_LENGTHS = (512, 2048, 8192, 16384, 32768, 65536)


def config(idx: int, L: Optional[int] = None, nthreads: Optional[int] = None) -> Workload:
    """Full-size workload `idx` (1..5).  Config 2 takes its cache length L."""
    seed = CONFIG_SEED_BASE + idx
    if idx == 1:
        return make_problem(1, 8, 8, 64, 512, seed, name="tiny-mha-L512", nthreads=nthreads)
    if idx == 2:
        L = 65536 if L is None else int(L)
        return make_problem(1, 64, 8, 128, L, seed, name=f"codellama34b-gqa8-L{L}",
                            nthreads=nthreads)
    if idx == 3:
        sl = uniform_int(stream_seed(seed, STREAM_SEQLENS), 32, 1024, 32768)
        return make_problem(32, 32, 8, 128, 32768, seed, seqlens=sl, nan_pad=True,
                            name="varlen-B32", nthreads=nthreads)
    if idx == 4:
        return make_problem(8, 32, 8, 128, 131072, seed, block_size=16,
                            name="paged-B8-L128K-bs16", nthreads=nthreads)
    if idx == 5:
        w = make_problem(1, 32, 8, 128, 262144, seed, name="peaked-L256K", nthreads=nthreads)
        plant_dominant_keys(w, 64, seed)
        return w
    raise ValueError(f"no workload {idx}")
