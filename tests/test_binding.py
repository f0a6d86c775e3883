"""Argument checks of the Python decode() (CPU only: every check raises
before the library is called, and the device check comes last)."""
import pytest
import torch

import split_kv_decode_attn_b200 as fd


def args(B=2, Hq=16, Hkv=2, D=128, L=256, dtype=torch.bfloat16):
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16)
    k = torch.zeros(B, Hkv, L, D, dtype=dtype)
    v = torch.zeros(B, Hkv, L, D, dtype=dtype)
    return q, k, v


def raises(match, *a, **kw):
    with pytest.raises(ValueError, match=match):
        fd.decode(*a, **kw)


def test_valid_cpu_tensors_stop_at_the_device_check():
    q, k, v = args()
    raises("CUDA device", q, k, v, torch.zeros(2, dtype=torch.int32))
    q8, k8, v8 = args(dtype=torch.uint8)
    raises("CUDA device", q8, k8, v8, k_scale=0.5, v_scale=0.5)


def test_dtypes():
    q, k, v = args()
    raises("q: dtype", q.float(), k, v)
    raises("k_cache: dtype", q, k.float(), v.float())
    raises("v_cache: dtype", q, k, v.to(torch.float16))
    raises("seqlens: dtype", q, k, v, torch.zeros(2, dtype=torch.int64))
    raises("out: dtype", q, k, v, out=torch.zeros(2, 16, 128))
    raises("lse: dtype", q, k, v, lse=torch.zeros(2, 16, dtype=torch.float64))


def test_shapes():
    q, k, v = args()
    raises("q: expected", q[0], k, v)
    raises("k_cache: expected 4", q, k[0], v[0])
    raises("v_cache: shape", q, k, v[:, :, :128].contiguous())
    raises("head dim", q[:, :, :64].contiguous(), k, v)
    raises("sequences", q[:1].contiguous(), k, v)
    raises("seqlens: shape", q, k, v, torch.zeros(3, dtype=torch.int32))
    raises("out: shape", q, k, v, out=torch.zeros(2, 16, 64, dtype=torch.bfloat16))
    raises("lse: shape", q, k, v, lse=torch.zeros(16, dtype=torch.float32))
    raises("max_len", q, k, v, max_len=512)      # more rows than the cache holds
    raises("max_len", q, k, v, max_len=128)      # would misplace the heads
    raises("kv_layout", q, k, v, kv_layout=2)


def test_paged_tables():
    q = torch.zeros(2, 16, 128, dtype=torch.bfloat16)
    pages = torch.zeros(8, 2, 16, 128, dtype=torch.bfloat16)
    raises("block_table: expected", q, pages, pages, block_table=torch.zeros(3, 4, dtype=torch.int32))
    raises("block_table: dtype", q, pages, pages, block_table=torch.zeros(2, 4, dtype=torch.int64))
    raises("CUDA device", q, pages, pages, block_table=torch.zeros(2, 4, dtype=torch.int32))


def test_views_that_are_not_contiguous():
    q, k, v = args()
    raises("q must be contiguous", q.transpose(0, 1).contiguous().transpose(0, 1), k, v)
    kt = torch.zeros(2, 256, 2, 128, dtype=torch.bfloat16).transpose(1, 2)   # [B, Hkv, L, D] view
    raises("k_cache must be contiguous", q, kt, kt)
    wide = torch.zeros(2, 2, 512, 128, dtype=torch.bfloat16)[:, :, :256]
    raises("k_cache must be contiguous", q, wide, wide)


def test_sharded_helpers_check_their_tensors():
    from split_kv_decode_attn_b200 import sharded
    q, k, v = args()
    with pytest.raises(ValueError, match="CUDA device"):
        sharded.local_partial(q, k, v, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="seqlens: dtype"):
        sharded.local_partial(q, k, v, torch.zeros(2, dtype=torch.int64))
    with pytest.raises(ValueError, match="float32"):
        sharded.combine(torch.zeros(2, 2, 16, 128, dtype=torch.float64), torch.zeros(2, 2, 16))
    P = sharded.packed_floats(2, 16, 128)
    with pytest.raises(ValueError, match="float32"):
        sharded.combine_packed(torch.zeros(2, P, dtype=torch.float64), 2, 16, 128)
    with pytest.raises(ValueError, match="parts shape"):
        sharded.combine_packed(torch.zeros(2, P - 64), 2, 16, 128)
    with pytest.raises(ValueError, match="contiguous"):
        sharded.combine_packed(torch.zeros(P, 2).t(), 2, 16, 128)
    with pytest.raises(ValueError, match="CUDA device"):
        sharded.combine_packed(torch.zeros(2, P), 2, 16, 128)
    with pytest.raises(ValueError, match="lse_all shape"):
        sharded.combine(torch.zeros(2, 2, 16, 128), torch.zeros(2, 16))
    with pytest.raises(ValueError, match="CUDA device"):
        sharded.combine(torch.zeros(2, 2, 16, 128), torch.zeros(2, 2, 16))


def test_static_workspace_wrapper_checks_its_tensors():
    """fd_decode_static_workspace takes the problem struct and raw tensors; a
    strided or padded cache, or a problem that does not describe the tensors,
    is rejected before the C call (which sees only addresses)."""
    q, k, v = args()
    prob = fd.make_problem(2, 16, 2, 128, 256)
    out = torch.zeros(2, 16, 128, dtype=torch.bfloat16)
    lse = torch.zeros(2, 16)

    def call(*a, prob=prob):
        with pytest.raises(ValueError) as e:
            fd.fd_decode_static_workspace(prob, *a, None, None, 0.125, 4, out, lse)
        return str(e.value)

    kt = torch.zeros(2, 256, 2, 128, dtype=torch.bfloat16).transpose(1, 2)
    assert "k_cache must be contiguous" in call(q, kt, kt)
    wide = torch.zeros(2, 2, 512, 128, dtype=torch.bfloat16)[:, :, :256]
    assert "k_cache must be contiguous" in call(q, wide, wide)
    padded = torch.zeros(2, 2, 512, 128, dtype=torch.bfloat16)
    assert "max_len" in call(q, padded, padded)
    assert "Hkv" in call(q, k, v, prob=fd.make_problem(2, 16, 4, 128, 256))
    assert "(B, Hq, D)" in call(q, k, v, prob=fd.make_problem(2, 32, 2, 128, 256))
    assert "CUDA device" in call(q, k, v)
