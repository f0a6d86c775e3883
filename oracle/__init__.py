"""fp64 CPU oracle of split-KV decode attention (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It is independent of the CUDA library: it imports
nothing from it and the two share no code.  The arithmetic lives in
``oracle.cpp`` (plain fp64 C++); this file only marshals numpy arrays.

Inputs are bf16 bit patterns held as ``numpy.uint16``; outputs are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
# A test may point the wrapper at a deliberately broken copy of the oracle
# (see tests/test_oracle_mutants.py) to prove that the pins catch it.
_LIB_OVERRIDE = os.environ.get("FD_ORACLE_LIB")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so next to it (plain g++, -O2, IEEE fp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-Wall", "-Wextra", "-shared",
                               "-fPIC", "-pthread", _SRC, "-o", _LIB])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            lib = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            lib = ctypes.CDLL(_LIB)
        vp, L, I, F = ctypes.c_void_p, ctypes.c_long, ctypes.c_int, ctypes.c_float
        lib.oracle_attend.argtypes = [L, I, I, vp, vp, vp, L, F, vp, vp]
        lib.oracle_attend.restype = None
        lib.oracle_attend_split.argtypes = [L, I, I, vp, vp, vp, L, F, L, vp, vp, vp, vp, L]
        lib.oracle_attend_split.restype = None
        lib.oracle_decode.argtypes = [I, I, I, I, L, vp, vp, vp, vp, F, vp, vp, I]
        lib.oracle_decode.restype = I
        lib.oracle_attend_f64.argtypes = [L, I, I, vp, vp, vp, L, ctypes.c_double, vp, vp]
        lib.oracle_attend_f64.restype = None
        _lib = lib
    return _lib


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def attend(q, k, v, scale: float):
    """G query heads sharing one KV head.

    q [G, D], k/v [n, D] (bf16 bits).  Returns (out [G, D] fp64, lse [G] fp64)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    G, D = q.shape
    n = k.shape[0]
    assert k.shape == (n, D) and v.shape == (n, D)
    out = np.empty((G, D), np.float64)
    lse = np.empty(G, np.float64)
    _load().oracle_attend(n, D, G, q.ctypes.data, k.ctypes.data, v.ctypes.data, D,
                          np.float32(scale), out.ctypes.data, lse.ctypes.data)
    return out, lse


def attend_f64(q, k, v, scale: float):
    """attend() on fp64 values (for caches whose real values are not bf16,
    such as dequantised fp8).  q [G, D], k/v [n, D] float64."""
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    G, D = q.shape
    n = k.shape[0]
    assert k.shape == (n, D) and v.shape == (n, D)
    out = np.empty((G, D), np.float64)
    lse = np.empty(G, np.float64)
    _load().oracle_attend_f64(n, D, G, q.ctypes.data, k.ctypes.data, v.ctypes.data, D,
                              float(scale), out.ctypes.data, lse.ctypes.data)
    return out, lse


def attend_split(q, k, v, scale: float, chunk: int, max_parts: int = 0):
    """Split-then-combine with chunk length `chunk`.

    Returns (out [G, D], lse [G]) and, when max_parts > 0, also the per-split
    partials (part_o [G, max_parts, D], part_lse [G, max_parts])."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    G, D = q.shape
    n = k.shape[0]
    assert chunk > 0
    out = np.empty((G, D), np.float64)
    lse = np.empty(G, np.float64)
    po = np.empty((G, max_parts, D), np.float64) if max_parts else None
    pl = np.empty((G, max_parts), np.float64) if max_parts else None
    _load().oracle_attend_split(n, D, G, q.ctypes.data, k.ctypes.data, v.ctypes.data, D,
                                np.float32(scale), chunk, out.ctypes.data, lse.ctypes.data,
                                po.ctypes.data if po is not None else None,
                                pl.ctypes.data if pl is not None else None, max_parts)
    if max_parts:
        return out, lse, po, pl
    return out, lse


def decode(q, k, v, scale: float, seqlens=None, nthreads: int = 0):
    """Whole batch over a contiguous cache.

    q [B, Hq, D]; k, v [B, Hkv, max_len, D]; seqlens [B] int32 or None.
    Returns (out [B, Hq, D], lse [B, Hq]) in fp64."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hq, D = q.shape
    _, Hkv, max_len, D2 = k.shape
    assert D2 == D and v.shape == k.shape and k.shape[0] == B
    sl = None
    if seqlens is not None:
        sl = np.ascontiguousarray(seqlens, dtype=np.int32)
        assert sl.shape == (B,)
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    nt = nthreads or (os.cpu_count() or 1)
    rc = _load().oracle_decode(B, Hq, Hkv, D, max_len, q.ctypes.data, k.ctypes.data,
                               v.ctypes.data, sl.ctypes.data if sl is not None else None,
                               np.float32(scale), out.ctypes.data, lse.ctypes.data, nt)
    if rc != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return out, lse
