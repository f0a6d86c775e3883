"""B200-native split-KV decode attention (Flash-Decoding).

Python binding of libfd.so.  Every function here marshals arguments for the C
ABI declared in ``include/fd.h`` and calls it; all arithmetic runs in the
library's CUDA kernels.  There is no fallback: if libfd.so is missing or a
call fails, an exception is raised.

The functions named ``fd_*`` mirror the C entry points one to one and take
raw device pointers (ints) or torch tensors.  ``decode`` is a convenience
wrapper that allocates the outputs and workspace with torch and calls
``fd_decode`` on the current stream.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfd.so")

FD_OK = 0
FD_ERR_INVALID_ARGUMENT = -1
FD_ERR_UNSUPPORTED = -2
FD_ERR_WORKSPACE = -3
FD_ERR_CUDA = -4
FD_ERR_DEVICE_TIMEOUT = -5

# Entry points declared in include/fd.h.
EXPORTS = ("fd_plan", "fd_plan_sm", "fd_plan_seqlens", "fd_plan_problem", "fd_split_chunk",
           "fd_effective_splits", "fd_workspace_bytes", "fd_decode",
           "fd_decode_partial", "fd_combine", "fd_combine_strided", "fd_quantize_keys",
           "fd_decode_sparse",
           "fd_decode_static_workspace", "fd_check_device_error",
           "fd_selftest_device_timeout", "fd_status_string")

# Mirrors FD_STATIC_WORKSPACE_BYTES in include/fd.h (a CPU test compares the two).
FD_STATIC_WORKSPACE_BYTES = 8 << 20


class FdError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {fd_status_string(status)} ({status})" if what
                         else f"{fd_status_string(status)} ({status})")


FD_LAYOUT_HND = 0  # cache [.., Hkv, tokens, D]
FD_LAYOUT_NHD = 1  # cache [.., tokens, Hkv, D]
FD_KV_BF16 = 0       # bf16 cache
FD_KV_FP8_E4M3 = 1   # fp8 e4m3 cache, real value = scale * code
FD_FP8_MMA_SYNC = 0     # fp8: codes converted to f16, mma.sync (default)
FD_FP8_MMA_TCGEN05 = 1  # fp8: tcgen05 kind::f8f6f4 on the codes in shared memory


class fd_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("D", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("kv_layout", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float), ("fp8_mma", ctypes.c_int32)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libfd.so (raises if it is not built: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; build it with __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        I, vp, sz, F = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
        lib.fd_plan.argtypes = [I] * 6
        lib.fd_plan.restype = I
        lib.fd_plan_sm.argtypes = [I] * 7
        lib.fd_plan_sm.restype = I
        lib.fd_plan_seqlens.argtypes = [I] * 7 + [vp]
        lib.fd_plan_seqlens.restype = I
        lib.fd_plan_problem.argtypes = [I, ctypes.POINTER(fd_problem), vp]
        lib.fd_plan_problem.restype = I
        lib.fd_split_chunk.argtypes = [I, I]
        lib.fd_split_chunk.restype = I
        lib.fd_effective_splits.argtypes = [I, I]
        lib.fd_effective_splits.restype = I
        lib.fd_workspace_bytes.argtypes = [I, I, I, I]
        lib.fd_workspace_bytes.restype = sz
        lib.fd_decode.argtypes = [ctypes.POINTER(fd_problem), vp, vp, vp, vp, vp, F, I, vp, vp,
                                  vp, sz, vp]
        lib.fd_decode.restype = I
        lib.fd_decode_partial.argtypes = [ctypes.POINTER(fd_problem), vp, vp, vp, vp, vp, F, I,
                                          vp, vp, vp, sz, vp]
        lib.fd_decode_partial.restype = I
        lib.fd_quantize_keys.argtypes = [ctypes.POINTER(fd_problem), vp, vp, vp, vp, vp]
        lib.fd_quantize_keys.restype = I
        lib.fd_decode_sparse.argtypes = [ctypes.POINTER(fd_problem), vp, vp, vp, vp, vp, vp, F,
                                         F, I, vp, vp, vp, vp, sz, vp]
        lib.fd_decode_sparse.restype = I
        lib.fd_combine.argtypes = [I, I, I, I, vp, vp, vp, vp, vp]
        lib.fd_combine.restype = I
        lib.fd_combine_strided.argtypes = [I, I, I, I, vp, sz, vp, sz, vp, vp, vp]
        lib.fd_combine_strided.restype = I
        lib.fd_decode_static_workspace.argtypes = [ctypes.POINTER(fd_problem), vp, vp, vp, vp,
                                                   vp, F, I, vp, vp, vp]
        lib.fd_decode_static_workspace.restype = I
        lib.fd_selftest_device_timeout.argtypes = [ctypes.c_uint, vp]
        lib.fd_selftest_device_timeout.restype = I
        lib.fd_check_device_error.argtypes = [vp]
        lib.fd_check_device_error.restype = I
        lib.fd_status_string.argtypes = [I]
        lib.fd_status_string.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def _ptr(x) -> Optional[int]:
    """Device address of a torch tensor, an int address, or None."""
    if x is None or x.__class__ is int:
        return x or None
    return x.data_ptr() or None


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


# ---- one-to-one mirrors of the C entry points --------------------------------

def fd_status_string(status: int) -> str:
    return load_library().fd_status_string(int(status)).decode()


def fd_plan(B: int, Hq: int, Hkv: int, D: int, max_len: int, block_size: int = 0) -> int:
    return int(load_library().fd_plan(B, Hq, Hkv, D, max_len, block_size))


def fd_plan_sm(num_sms: int, B: int, Hq: int, Hkv: int, D: int, max_len: int,
               block_size: int = 0) -> int:
    return int(load_library().fd_plan_sm(num_sms, B, Hq, Hkv, D, max_len, block_size))


def fd_plan_seqlens(num_sms: int, B: int, Hq: int, Hkv: int, D: int, max_len: int,
                    block_size: int, seqlens) -> int:
    """Length-aware planner; `seqlens` is a host sequence of B ints (0 or a
    negative num_sms plans for the current device)."""
    import numpy as np
    sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    return int(load_library().fd_plan_seqlens(num_sms, B, Hq, Hkv, D, max_len, block_size,
                                              sl.ctypes.data))


def fd_plan_problem(num_sms: int, prob: "fd_problem", seqlens=None) -> int:
    """Planner for a whole problem (element type included); `seqlens` is a
    host sequence of B ints or None (every sequence holds max_len)."""
    import numpy as np
    sl = None if seqlens is None else np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    return int(load_library().fd_plan_problem(num_sms, ctypes.byref(prob),
                                              None if sl is None else sl.ctypes.data))


def fd_split_chunk(max_len: int, num_splits: int) -> int:
    return int(load_library().fd_split_chunk(max_len, num_splits))


def fd_effective_splits(max_len: int, num_splits: int) -> int:
    return int(load_library().fd_effective_splits(max_len, num_splits))


def fd_workspace_bytes(B: int, Hq: int, D: int, num_splits: int) -> int:
    return int(load_library().fd_workspace_bytes(B, Hq, D, num_splits))


def fd_decode(problem: fd_problem, q, k_cache, v_cache, seqlens, block_table, scale: float,
              num_splits: int, out, lse, workspace, workspace_bytes: int, stream=None) -> int:
    """Call the C fd_decode; returns its status code.  Tensor arguments may be
    torch tensors, int device addresses or None; `stream` a torch stream, an
    int cudaStream_t or None (torch's current stream)."""
    f = _lib.fd_decode if _lib is not None else load_library().fd_decode
    return f(ctypes.byref(problem), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
             _ptr(block_table), scale, num_splits, _ptr(out), _ptr(lse), _ptr(workspace),
             workspace_bytes, _stream(stream))


def fd_decode_partial(problem: fd_problem, q, k_cache, v_cache, seqlens, block_table,
                      scale: float, num_splits: int, out_f32, lse, workspace,
                      workspace_bytes: int, stream=None) -> int:
    """Call the C fd_decode_partial: exact attention over this shard of the
    history as fp32 output and lse, for fd_combine.  Returns the status."""
    return int(load_library().fd_decode_partial(
        ctypes.byref(problem), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
        _ptr(block_table), scale, num_splits, _ptr(out_f32), _ptr(lse), _ptr(workspace),
        workspace_bytes, _stream(stream)))


def fd_quantize_keys(problem: fd_problem, k_cache, seqlens, k8, k8_scale, stream=None) -> int:
    """Call the C fd_quantize_keys: int8 key codes and per-64-token-block
    scales for fd_decode_sparse.  Returns the status."""
    return int(load_library().fd_quantize_keys(ctypes.byref(problem), _ptr(k_cache),
                                               _ptr(seqlens), _ptr(k8), _ptr(k8_scale),
                                               _stream(stream)))


def fd_decode_sparse(problem: fd_problem, q, k_cache, v_cache, k8, k8_scale, seqlens,
                     scale: float, delta: float, num_splits: int, out, lse, kept, workspace,
                     workspace_bytes: int, stream=None) -> int:
    """Call the C fd_decode_sparse: the low-bit scan and top-delta block
    selection, then exact attention over the kept blocks.  Returns the status."""
    return int(load_library().fd_decode_sparse(
        ctypes.byref(problem), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k8), _ptr(k8_scale),
        _ptr(seqlens), scale, delta, num_splits, _ptr(out), _ptr(lse), _ptr(kept),
        _ptr(workspace), workspace_bytes, _stream(stream)))


def fd_combine(R: int, B: int, Hq: int, D: int, part_o, part_lse, out, lse, stream=None) -> int:
    """Call the C fd_combine: merge R partials [R, B, Hq, D] / [R, B, Hq].
    Returns the status."""
    return int(load_library().fd_combine(R, B, Hq, D, _ptr(part_o), _ptr(part_lse), _ptr(out),
                                         _ptr(lse), _stream(stream)))


def fd_combine_strided(R: int, B: int, Hq: int, D: int, part_o, o_stride: int, part_lse,
                       lse_stride: int, out, lse, stream=None) -> int:
    """Call the C fd_combine_strided: merge R partials placed at strides
    (counted in floats), e.g. R packed per-rank buffers gathered end to end.
    Returns the status."""
    return int(load_library().fd_combine_strided(R, B, Hq, D, _ptr(part_o), o_stride,
                                                 _ptr(part_lse), lse_stride, _ptr(out),
                                                 _ptr(lse), _stream(stream)))


def fd_decode_static_workspace(problem: fd_problem, q, k_cache, v_cache, seqlens, block_table,
                               scale: float, num_splits: int, out, lse, stream=None) -> int:
    """Call the C fd_decode_static_workspace: fd_decode for callers that cannot
    allocate device memory; its scratch is the library's static device array
    of FD_STATIC_WORKSPACE_BYTES.  Returns the status code.

    When q is a torch tensor, the tensors are checked as decode() checks them
    (dtype, shape, contiguity, device, and a contiguous cache's row count
    against problem.max_len) and against the problem's sizes, and a mismatch
    raises ValueError before anything is launched: the C ABI sees only
    addresses, and a strided or padded view would be read as dense memory."""
    if q is not None and q.__class__ is not int:
        if q.dim() == 3 and k_cache.dim() == 4:
            _check_problem_sizes(problem, q, k_cache)
        _check_decode_args(q, k_cache, v_cache, seqlens, block_table, problem.kv_layout,
                           problem.max_len if problem.block_size == 0 else None, out, lse, None)
    return int(load_library().fd_decode_static_workspace(
        ctypes.byref(problem), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
        _ptr(block_table), ctypes.c_float(scale), int(num_splits), _ptr(out), _ptr(lse),
        _stream(stream)))


def fd_check_device_error(stream=None) -> int:
    return int(load_library().fd_check_device_error(_stream(stream)))


def fd_selftest_device_timeout(limit_us: int, stream=None) -> int:
    return int(load_library().fd_selftest_device_timeout(int(limit_us), _stream(stream)))


# ---- convenience wrapper -----------------------------------------------------

def make_problem(B, Hq, Hkv, D, max_len, block_size=0, num_blocks=0, max_blocks_per_seq=0,
                 kv_layout=FD_LAYOUT_HND, kv_dtype=FD_KV_BF16, k_scale=1.0, v_scale=1.0,
                 fp8_mma=0):
    return fd_problem(B, Hq, Hkv, D, max_len, block_size, num_blocks, max_blocks_per_seq,
                      kv_layout, kv_dtype, k_scale, v_scale, fp8_mma)


def _check(t, name, dtypes, shape=None):
    """Checks a tensor argument of decode() before its address is passed on:
    the kernels read and write dense row-major buffers of the stated shapes."""
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def _check_decode_args(q, k_cache, v_cache, seqlens, block_table, kv_layout, max_len, out, lse,
                       workspace):
    """Shape, dtype, layout and device checks of decode(); raises ValueError.
    The device checks come last."""
    import torch
    cache_types = [torch.bfloat16, torch.uint8]
    if hasattr(torch, "float8_e4m3fn"):
        cache_types.append(torch.float8_e4m3fn)
    if q.dim() != 3:
        raise ValueError(f"q: expected [B, Hq, D], got shape {tuple(q.shape)}")
    B, Hq, D = q.shape
    _check(q, "q", [torch.bfloat16])
    if kv_layout not in (FD_LAYOUT_HND, FD_LAYOUT_NHD):
        raise ValueError(f"kv_layout: {kv_layout}, expected FD_LAYOUT_HND or FD_LAYOUT_NHD")
    if k_cache.dim() != 4:
        raise ValueError(f"k_cache: expected 4 dimensions, got shape {tuple(k_cache.shape)}")
    _check(k_cache, "k_cache", cache_types)
    _check(v_cache, "v_cache", [k_cache.dtype], k_cache.shape)
    if k_cache.shape[3] != D:
        raise ValueError(f"k_cache: head dim {k_cache.shape[3]}, q has {D}")
    if block_table is None:
        if k_cache.shape[0] != B:
            raise ValueError(f"k_cache: {k_cache.shape[0]} sequences, q has {B}")
        rows = k_cache.shape[2] if kv_layout == FD_LAYOUT_HND else k_cache.shape[1]
        if max_len is not None and max_len != rows:
            raise ValueError(f"max_len {max_len}: a contiguous cache holds {rows} rows per "
                             "sequence and KV head, and max_len must equal it")
    else:
        if block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError(f"block_table: expected [B={B}, max_blocks], got "
                             f"{tuple(block_table.shape)}")
        _check(block_table, "block_table", [torch.int32])
    if seqlens is not None:
        _check(seqlens, "seqlens", [torch.int32], (B,))
    if out is not None:
        _check(out, "out", [torch.bfloat16], (B, Hq, D))
    if lse is not None:
        _check(lse, "lse", [torch.float32], (B, Hq))
    if workspace is not None:
        _check(workspace, "workspace", None)
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("seqlens", seqlens),
                    ("block_table", block_table), ("out", out), ("lse", lse),
                    ("workspace", workspace)):
        if t is not None and (not t.is_cuda or t.device != q.device):
            raise ValueError(f"{name} is on {t.device}; every tensor must be on q's CUDA device "
                             f"({q.device})")


def _check_problem_sizes(problem: fd_problem, q, k_cache):
    """The problem's B, Hq, D, Hkv (and page size) must describe the tensors."""
    B, Hq, D = q.shape
    if (problem.B, problem.Hq, problem.D) != (B, Hq, D):
        raise ValueError(f"problem (B, Hq, D) = {(problem.B, problem.Hq, problem.D)}, q has "
                         f"{(B, Hq, D)}")
    hnd = problem.kv_layout == FD_LAYOUT_HND
    Hkv = k_cache.shape[1] if hnd else k_cache.shape[2]
    if problem.Hkv != Hkv:
        raise ValueError(f"problem Hkv = {problem.Hkv}, the cache holds {Hkv} KV heads")
    if problem.block_size:
        bs = k_cache.shape[2] if hnd else k_cache.shape[1]
        if (problem.block_size, problem.num_blocks) != (bs, k_cache.shape[0]):
            raise ValueError(f"problem pages {(problem.num_blocks, problem.block_size)}, the "
                             f"cache holds {(k_cache.shape[0], bs)}")


def decode(q, k_cache, v_cache, seqlens=None, block_table=None, *, max_len: Optional[int] = None,
           kv_layout: int = FD_LAYOUT_HND, scale: Optional[float] = None,
           num_splits: Optional[int] = None, out=None, lse=None, workspace=None, stream=None,
           k_scale: float = 1.0, v_scale: float = 1.0, fp8_mma: int = FD_FP8_MMA_SYNC):
    """Decode attention on torch CUDA tensors.

    q [B, Hq, D] bf16.  Caches: bf16, or E4M3 codes (torch.uint8 or
    torch.float8_e4m3fn, D = 128) whose real values are k_scale * code and
    v_scale * code.  FD_LAYOUT_HND contiguous [B, Hkv, max_len, D] or paged
    [num_blocks, Hkv, block_size, D]; FD_LAYOUT_NHD contiguous
    [B, max_len, Hkv, D] or paged [num_blocks, block_size, Hkv, D].  Paged
    caches come with block_table [B, max_blocks] int32.  seqlens [B] int32
    or None.  Returns (out [B, Hq, D] bf16, lse [B, Hq] fp32).  num_splits
    defaults to fd_plan_problem's choice.  fp8_mma picks the tensor-core path
    of an fp8 cache (FD_FP8_MMA_SYNC or FD_FP8_MMA_TCGEN05).  Raises
    ValueError for tensors of the wrong dtype, shape or device, or not
    contiguous, before anything is launched, and FdError for a failing
    status."""
    import torch
    _check_decode_args(q, k_cache, v_cache, seqlens, block_table, kv_layout, max_len, out, lse,
                       workspace)
    B, Hq, D = q.shape
    block_size = 0
    fp8 = k_cache.element_size() == 1
    kv_dtype = FD_KV_FP8_E4M3 if fp8 else FD_KV_BF16
    if block_table is None:
        if kv_layout == FD_LAYOUT_HND:
            _, Hkv, L, _ = k_cache.shape
        else:
            _, L, Hkv, _ = k_cache.shape
        max_len = L if max_len is None else max_len
        prob = make_problem(B, Hq, Hkv, D, max_len, kv_layout=kv_layout, kv_dtype=kv_dtype,
                            k_scale=k_scale, v_scale=v_scale, fp8_mma=fp8_mma)
    else:
        if kv_layout == FD_LAYOUT_HND:
            nb, Hkv, bs, _ = k_cache.shape
        else:
            nb, bs, Hkv, _ = k_cache.shape
        block_size = bs
        mbps = block_table.shape[1]
        max_len = mbps * bs if max_len is None else max_len
        prob = make_problem(B, Hq, Hkv, D, max_len, bs, nb, mbps, kv_layout, kv_dtype, k_scale,
                            v_scale, fp8_mma)
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    if num_splits is None:
        num_splits = fd_plan_problem(0, prob)
        if num_splits < 0:
            raise FdError(num_splits, "fd_plan_problem")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    wbytes = fd_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None and wbytes:
        workspace = torch.empty(wbytes // 4, dtype=torch.float32, device=q.device)
    have = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = fd_decode(prob, q, k_cache, v_cache, seqlens, block_table, scale, num_splits, out, lse,
                   workspace, have, stream)
    if st != FD_OK:
        raise FdError(st, "fd_decode")
    return out, lse
