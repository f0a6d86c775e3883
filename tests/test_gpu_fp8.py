"""GPU parity of the fp8 e4m3 KV-cache path against the fp64 oracle.

The oracle sees the dequantised cache (k_scale * code, v_scale * code, exact
in fp64) and the bf16 queries; the default path multiplies the codes in f16 on
the tensor cores, the tcgen05 path multiplies them as e4m3 with q and the
weights split into e4m3 codes; both apply the scales in fp32.  Same tolerances as the bf16
path.  Covers every group size, ragged lengths with NaN-coded padding, forced
split counts, paged versus contiguous and token-major versus head-major bit
identity, determinism, unequal non-power-of-two scales and a long context."""
import dataclasses

import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import OnDevice, assert_close, free_device, reference, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_device):
    yield
    free_device()


# Both tensor-core paths of an fp8 cache: the default (codes converted to f16,
# mma.sync) and tcgen05 (kind::f8f6f4 on the codes; taken for G in {2, 4, 8}
# on grids of at most one CTA per SM, the default path elsewhere).
@pytest.fixture(params=[fd.FD_FP8_MMA_SYNC, fd.FD_FP8_MMA_TCGEN05], ids=["mma_sync", "tcgen05"])
def mma(request):
    return request.param


def contiguous_copy(p: wl.Workload) -> wl.Workload:
    """The same logical fp8 cache as a contiguous [B, Hkv, L, D] array."""
    kc = np.zeros((p.B, p.Hkv, p.max_len, p.D), np.uint8)
    vc = np.zeros_like(kc)
    for b in range(p.B):
        for h in range(p.Hkv):
            k, v = p.logical_kv(b, h)
            kc[b, h, :len(k)] = k
            vc[b, h, :len(v)] = v
    return dataclasses.replace(p, name="contig", k=kc, v=vc, block_table=None, block_size=0,
                               layout="HND")


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_fp8_group_sizes_and_ragged_lengths(G, mma):
    Hkv = 2
    lens = [0, 1, 63, 64, 65, 200, 777, 2000]
    w = wl.make_problem(len(lens), G * Hkv, Hkv, 128, 2000, seed=300 + G, seqlens=lens,
                        nan_pad=True, kv_dtype="fp8")
    d = OnDevice(w, mma)
    ref, rl = reference(w)
    for S in (1, 2, 3, 7, 16, 32):
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"fp8 G={G} S={S}")


@pytest.mark.parametrize("G", [1, 8, 16])
def test_fp8_long_splits_at_one_cta_per_sm_ragged(G, mma):
    """fp8 splits of more than 64 tiles on a grid of at most one CTA per SM
    (eight consumer warps, 8-stage ring), ragged lengths and NaN codes past
    every length; and splits of at most 64 tiles (12-stage ring)."""
    Hkv = 2
    lens = [0, 1, 4097, 5000, 9000]
    w = wl.make_problem(len(lens), G * Hkv, Hkv, 128, 9000, seed=310 + G, seqlens=lens,
                        nan_pad=True, kv_dtype="fp8")
    d = OnDevice(w, mma)
    ref, rl = reference(w)
    for S in (1, 2, 3):     # 141, 71 and 47 tiles per split
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"fp8 long splits G={G} S={S}")


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("bs", [16, 64, 256])
def test_fp8_paged_matches_contiguous_bit_for_bit(bs, layout, mma):
    B, Hq, Hkv, L = 3, 64, 8, 1024
    p = wl.make_problem(B, Hq, Hkv, 128, L, seed=340 + bs, seqlens=[1024, 517, 64],
                        block_size=bs, num_blocks=B * L // bs + 3, layout=layout,
                        kv_dtype="fp8")
    c = contiguous_copy(p)
    dp, dc = OnDevice(p, mma), OnDevice(c, mma)
    ref, rl = reference(c)
    for S in (1, 5):
        gp, lp, _ = run_gpu(dp, S)
        gc_, lc, _ = run_gpu(dc, S)
        assert_close(gp, lp, ref, rl, f"fp8 paged {layout} bs={bs} S={S}")
        assert np.array_equal(gp, gc_) and np.array_equal(lp, lc)


@pytest.mark.parametrize("bs", [8, 32])
def test_fp8_paged_sixteen_heads_per_group(bs, mma):
    """G = 16 (two column blocks) on a paged fp8 cache, pages under a tile."""
    B, Hkv, L = 2, 2, 512
    p = wl.make_problem(B, 16 * Hkv, Hkv, 128, L, seed=350 + bs, seqlens=[512, 77],
                        block_size=bs, num_blocks=B * L // bs + 2, kv_dtype="fp8")
    c = contiguous_copy(p)
    dp, dc = OnDevice(p, mma), OnDevice(c, mma)
    ref, rl = reference(c)
    for S in (1, 3):
        gp, lp, _ = run_gpu(dp, S)
        gc_, lc, _ = run_gpu(dc, S)
        assert_close(gp, lp, ref, rl, f"fp8 paged G=16 bs={bs} S={S}")
        assert np.array_equal(gp, gc_) and np.array_equal(lp, lc)


def test_fp8_token_major_matches_head_major(mma):
    B, Hkv, L = 3, 4, 1500
    n = wl.make_problem(B, 16 * Hkv // 4, Hkv, 128, L, seed=360, seqlens=[1500, 9, 640],
                        nan_pad=True, layout="NHD", kv_dtype="fp8")
    h = dataclasses.replace(n, name="hnd", layout="HND",
                            k=np.ascontiguousarray(n.k.transpose(0, 2, 1, 3)),
                            v=np.ascontiguousarray(n.v.transpose(0, 2, 1, 3)))
    dn, dh = OnDevice(n, mma), OnDevice(h, mma)
    ref, rl = reference(h)
    for S in (1, 6):
        gn, ln_, _ = run_gpu(dn, S)
        gh, lh, _ = run_gpu(dh, S)
        assert_close(gn, ln_, ref, rl, f"fp8 NHD S={S}")
        assert np.array_equal(gn, gh) and np.array_equal(ln_, lh)


@pytest.mark.parametrize("G", [2, 8])
def test_fp8_running_maximum_jumps(G, mma):
    """Keys planted along the sequence raise the running maximum by several
    nats at a time (about 6 per step for the group's heads), in tiles that
    alternate between the two sets of warps: the one-CTA-per-SM fp8 kernel
    keeps its weights relative to an older maximum until the maximum has
    grown by more than 2^8 and then rescales its accumulators.  The earlier
    tokens keep a weight that still counts, so a missed or doubled rescale
    shows in the output."""
    Hkv = 2
    w = wl.make_problem(2, G * Hkv, Hkv, 128, 6000, seed=396 + G, seqlens=[6000, 3001],
                        kv_dtype="fp8")
    positions = [100, 900, 2000, 3500, 5100]
    for b in range(w.B):
        for h in range(Hkv):
            u = wl.bf16_bits_to_f64(w.q[b, h * G:(h + 1) * G]).sum(axis=0)
            u /= np.linalg.norm(u)
            for i, pos in enumerate(positions):
                mag = (2.0 + 1.6 * i) * np.sqrt(G / 8.0)
                key = np.clip(mag * u * np.sqrt(w.D) / w.k_scale, -440.0, 440.0)
                w.k[b, h, pos, :] = wl.f64_to_e4m3_bits(key)
    d = OnDevice(w, mma)
    ref, rl = reference(w)
    for S in (1, 2, 3):
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"fp8 max jumps G={G} S={S}")


def test_fp8_unequal_scales(mma):
    w = wl.make_problem(2, 32, 4, 128, 3000, seed=370, seqlens=[3000, 1234], kv_dtype="fp8")
    w = dataclasses.replace(w, k_scale=0.0217, v_scale=0.0461)
    d = OnDevice(w, mma)
    ref, rl = reference(w)
    for S in (1, 4, 11):
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"fp8 scales S={S}")


def test_fp8_single_token_returns_scaled_v0_exactly(mma):
    w = wl.make_problem(2, 16, 2, 128, 64, seed=380, seqlens=[1, 1], kv_dtype="fp8")
    d = OnDevice(w, mma)
    got, _, _ = run_gpu(d, 1)
    for b in range(2):
        for h in range(16):
            v0 = w.v_scale * wl.e4m3_bits_to_f64(w.v[b, h // w.G, 0])
            assert np.array_equal(got[b, h], v0)


def test_fp8_repeated_runs_are_bit_identical(mma):
    w = wl.make_problem(2, 64, 8, 128, 5000, seed=390, seqlens=[5000, 2999], kv_dtype="fp8")
    d = OnDevice(w, mma)
    for S in (1, 9):
        a, la, _ = run_gpu(d, S)
        for _ in range(2):
            b, lb, _ = run_gpu(d, S)
            assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_fp8_codellama34b_shape_long_context(mma):
    """B=1, Hq=64, Hkv=8, L=65536 in the planner's split count; the oracle
    computes two KV heads (16 query rows)."""
    w = wl.make_problem(1, 64, 8, 128, 65536, seed=395, kv_dtype="fp8")
    d = OnDevice(w, mma)
    got, gl, S = run_gpu(d)
    ref, rl = reference(w, groups=[(0, 0), (0, 5)])
    e = assert_close(got, gl, ref, rl, f"fp8 L=64K S={S}")
    print(f"fp8 64K planner S={S} errors {e}")


def test_fp8_tcgen05_path_runs_its_own_arithmetic():
    """On a grid of one CTA per SM with G = 8 the tcgen05 path runs its own
    kernel: both paths match the oracle, and their outputs differ in the
    last bits (the mma.sync path rounds q and the weights to f16, the tcgen05
    path splits them into e4m3 codes)."""
    w = wl.make_problem(1, 64, 8, 128, 8192, seed=398, kv_dtype="fp8")
    ref, rl = reference(w, groups=[(0, 0), (0, 7)])
    res = {}
    for m in (fd.FD_FP8_MMA_SYNC, fd.FD_FP8_MMA_TCGEN05):
        got, gl, S = run_gpu(OnDevice(w, m), 16)
        assert_close(got, gl, ref, rl, f"fp8 mma={m} S={S}")
        res[m] = (got, gl)
    a, b = res[fd.FD_FP8_MMA_SYNC], res[fd.FD_FP8_MMA_TCGEN05]
    assert not (np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]))


def test_fp8_decode_wrapper(mma):
    """The torch-level decode() on uint8 code tensors, with the path chosen
    by its fp8_mma argument, against the oracle."""
    import torch
    w = wl.make_problem(2, 16, 2, 128, 3000, seed=399, seqlens=[3000, 1700], kv_dtype="fp8")
    dev = torch.device("cuda", torch.cuda.current_device())
    q = torch.from_numpy(w.q.view(np.int16)).to(dev).view(torch.bfloat16)
    k = torch.from_numpy(w.k).to(dev)
    v = torch.from_numpy(w.v).to(dev)
    sl = torch.from_numpy(w.seqlens).to(dev)
    out, lse = fd.decode(q, k, v, sl, scale=w.scale, num_splits=6, k_scale=w.k_scale,
                         v_scale=w.v_scale, fp8_mma=mma)
    torch.cuda.synchronize()
    assert fd.fd_check_device_error() == fd.FD_OK
    got = wl.bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))
    ref, rl = reference(w)
    assert_close(got, lse.cpu().numpy().astype(np.float64), ref, rl, f"fp8 decode() mma={mma}")
