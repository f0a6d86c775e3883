"""GPU parity of fd_decode (called through the C ABI) against the fp64 oracle
on the same seeded bf16 inputs.

Covers the five workload shapes at full size in the launch configuration the
benchmark times (planner-chosen split count), forced split counts, every
supported group size and head dim, ragged and empty sequences, every paged
block size, bit-exact determinism, paged-versus-contiguous identity, closed
forms, canaries around the outputs and workspace, and error codes with real
device pointers."""
import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import (OnDevice, assert_close, big_outputs, free_device, host_bf16, reference,
                    run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_device):
    yield
    free_device()


# ---- the five workloads -------------------------------------------------------

@pytest.mark.parametrize("S", [1, 2, 4, 8])
def test_tiny_mha_all_split_counts(S):
    w = wl.config(1)
    d = OnDevice(w)
    got, gl, _ = run_gpu(d, S)
    ref, rl = reference(w)
    assert_close(got, gl, ref, rl, f"tiny S={S}")


@pytest.mark.parametrize("L", wl.CONFIG2_LENGTHS)
def test_codellama34b_shape_planner_splits(L):
    w = wl.config(2, L=L)
    d = OnDevice(w)
    ref, rl = reference(w)
    got, gl, S = run_gpu(d)
    e = assert_close(got, gl, ref, rl, f"L={L} S={S}")
    assert big_outputs(ref) == 0
    print(f"L={L} planner S={S} max|dO|={e[0]:.2e} max|dlse|={e[1]:.2e}")
    if L <= 8192:
        got1, gl1, _ = run_gpu(d, 1)
        assert_close(got1, gl1, ref, rl, f"L={L} S=1")


def test_varlen_batch_with_nan_padding():
    w = wl.config(3)
    d = OnDevice(w)
    got, gl, S = run_gpu(d)
    ref, rl = reference(w)
    e = assert_close(got, gl, ref, rl, f"varlen S={S}")
    print(f"varlen planner S={S} errors {e}")
    for S2 in (1, 8, 24):
        got2, gl2, _ = run_gpu(d, S2)
        assert_close(got2, gl2, ref, rl, f"varlen S={S2}")


def test_paged_cache_block16():
    w = wl.config(4)
    d = OnDevice(w)
    got, gl, S = run_gpu(d)
    # every (sequence, KV head) group of 4 query heads, from logical order
    ref, rl = reference(w)
    e = assert_close(got, gl, ref, rl, f"paged S={S}")
    print(f"paged planner S={S} errors {e}")


def test_long_context_peaked_softmax():
    w = wl.config(5)
    d = OnDevice(w)
    got, gl, S = run_gpu(d)
    ref, rl = reference(w)
    e = assert_close(got, gl, ref, rl, f"peaked S={S}")
    # the aligned heads (first of each group) are dominated by the planted keys
    assert np.all(rl[0, ::w.G] > 40.0)
    print(f"peaked planner S={S} errors {e} lse range {rl.min():.2f}..{rl.max():.2f}")
    got1, gl1, _ = run_gpu(d, 1)
    assert_close(got1, gl1, ref, rl, "peaked S=1")


# ---- shapes, ragged lengths, split counts ------------------------------------

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_group_sizes_and_ragged_lengths(G, D):
    Hkv = 2
    lens = [0, 1, 63, 64, 65, 200, 777, 2000]
    w = wl.make_problem(len(lens), G * Hkv, Hkv, D, 2000, seed=100 + G * D, seqlens=lens,
                        nan_pad=True)
    d = OnDevice(w)
    ref, rl = reference(w)
    for S in (1, 2, 3, 7, 16, 32):
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"G={G} D={D} S={S}")


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_long_splits_at_one_cta_per_sm_ragged(G):
    """Splits of more than 64 tiles on a grid of at most one CTA per SM: the
    eight consumer warps over the shorter ring, with ragged lengths, an
    empty sequence and NaN padding past every length."""
    Hkv = 2
    lens = [0, 1, 4097, 5000, 9000]
    w = wl.make_problem(len(lens), G * Hkv, Hkv, 128, 9000, seed=150 + G, seqlens=lens,
                        nan_pad=True)
    d = OnDevice(w)
    ref, rl = reference(w)
    for S in (1, 2):        # 141 and 71 tiles per split, 10 and 20 CTAs
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"long splits G={G} S={S}")


def test_all_sequences_empty():
    w = wl.make_problem(3, 16, 2, 128, 500, seed=5, seqlens=[0, 0, 0])
    d = OnDevice(w)
    for S in (1, 4):
        got, gl, _ = run_gpu(d, S)
        assert np.all(got == 0) and np.all(np.isneginf(gl))


def test_zero_length_cache():
    import torch
    w = wl.make_problem(2, 8, 8, 64, 0, seed=6)
    d = OnDevice(w)
    # nothing is read from a zero-length cache, but the pointers must be valid
    d.k = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    d.v = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    got, gl, _ = run_gpu(d, 1)
    assert np.all(got == 0) and np.all(np.isneginf(gl))


def test_seqlens_are_clamped():
    w = wl.make_problem(2, 8, 2, 128, 300, seed=8, seqlens=[1000, -5])
    d = OnDevice(w)
    ref, rl = reference(w)  # the oracle clamps the same way
    for S in (1, 3):
        got, gl, _ = run_gpu(d, S)
        assert_close(got, gl, ref, rl, f"clamp S={S}")


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128, 256])
def test_paged_block_sizes_match_contiguous_bit_for_bit(bs, layout):
    B, Hq, Hkv, D, L = 3, 32, 8, 128, 1024
    lens = [1024, 517, 64]
    p = wl.make_problem(B, Hq, Hkv, D, L, seed=40 + bs, seqlens=lens, block_size=bs,
                        num_blocks=B * L // bs + 5, layout=layout)
    # the same logical cache, contiguous
    kc = np.zeros((B, Hkv, L, D), np.uint16)
    vc = np.zeros((B, Hkv, L, D), np.uint16)
    for b in range(B):
        for h in range(Hkv):
            k, v = p.logical_kv(b, h)
            kc[b, h, :len(k)] = k
            vc[b, h, :len(v)] = v
    c = wl.Workload(name="contig", B=B, Hq=Hq, Hkv=Hkv, D=D, max_len=L, q=p.q, k=kc, v=vc,
                    scale=p.scale, seqlens=p.seqlens)
    dp, dc = OnDevice(p), OnDevice(c)
    ref, rl = reference(c)
    for S in (1, 5):
        gp, lp, _ = run_gpu(dp, S)
        gc_, lc, _ = run_gpu(dc, S)
        assert_close(gp, lp, ref, rl, f"paged {layout} bs={bs} S={S}")
        assert np.array_equal(gp, gc_) and np.array_equal(lp, lc)


@pytest.mark.parametrize("D,G", [(128, 8), (128, 4), (64, 1)])
def test_token_major_contiguous_cache(D, G):
    """[B, max_len, Hkv, D] gives the same bits as [B, Hkv, max_len, D]."""
    B, Hkv, L = 4, 4, 1500
    lens = [1500, 1, 640, 0]
    n = wl.make_problem(B, G * Hkv, Hkv, D, L, seed=60 + G, seqlens=lens, nan_pad=True,
                        layout="NHD")
    h = wl.Workload(name="hnd", B=B, Hq=n.Hq, Hkv=Hkv, D=D, max_len=L, q=n.q,
                    k=np.ascontiguousarray(n.k.transpose(0, 2, 1, 3)),
                    v=np.ascontiguousarray(n.v.transpose(0, 2, 1, 3)),
                    scale=n.scale, seqlens=n.seqlens)
    dn, dh = OnDevice(n), OnDevice(h)
    ref, rl = reference(h)
    for S in (1, 5, 32):
        gn, ln_, _ = run_gpu(dn, S)
        gh, lh, _ = run_gpu(dh, S)
        assert_close(gn, ln_, ref, rl, f"NHD D={D} G={G} S={S}")
        assert np.array_equal(gn, gh) and np.array_equal(ln_, lh)


# ---- determinism, closed forms, buffers ----------------------------------------

def test_repeated_runs_are_bit_identical():
    w = wl.make_problem(4, 32, 8, 128, 5000, seed=9, seqlens=[5000, 4000, 1, 2999])
    d = OnDevice(w)
    for S in (1, 6, 37):
        a, la, _ = run_gpu(d, S)
        for _ in range(3):
            b, lb, _ = run_gpu(d, S)
            assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_single_token_returns_v0_exactly():
    w = wl.make_problem(2, 16, 2, 128, 64, seed=10, seqlens=[1, 1])
    d = OnDevice(w)
    got, gl, _ = run_gpu(d, 1)
    G = w.G
    for b in range(2):
        for h in range(16):
            v0 = wl.bf16_bits_to_f64(w.v[b, h // G, 0])
            assert np.array_equal(got[b, h], v0)


def test_zero_query_gives_mean_of_v():
    w = wl.make_problem(1, 8, 1, 128, 3000, seed=11)
    w.q[:] = 0
    d = OnDevice(w)
    vmean = wl.bf16_bits_to_f64(w.v[0, 0]).mean(axis=0)
    for S in (1, 9):
        got, gl, _ = run_gpu(d, S)
        assert np.max(np.abs(got[0] - vmean[None, :])) <= 1e-2
        assert np.max(np.abs(gl - np.log(3000))) <= 1e-3


def test_outputs_and_workspace_stay_in_bounds():
    import torch
    w = wl.make_problem(2, 16, 2, 128, 700, seed=12, seqlens=[700, 333])
    d = OnDevice(w)
    S = 5
    need = fd.fd_workspace_bytes(w.B, w.Hq, w.D, S)
    pad = 4096
    out_buf = torch.full((2 * pad + w.B * w.Hq * w.D,), 7.0, dtype=torch.bfloat16, device="cuda")
    lse_buf = torch.full((2 * pad + w.B * w.Hq,), 7.0, dtype=torch.float32, device="cuda")
    ws_buf = torch.full(((need + 2 * 4 * pad) // 4,), 7.0, dtype=torch.float32, device="cuda")
    out = out_buf[pad:pad + w.B * w.Hq * w.D]
    lse = lse_buf[pad:pad + w.B * w.Hq]
    ws = ws_buf[pad:]
    st = fd.fd_decode(d.problem(), d.q, d.k, d.v, d.seqlens, None, w.scale, S, out, lse, ws,
                      need, None)
    assert st == fd.FD_OK
    torch.cuda.synchronize()
    assert torch.all(out_buf[:pad] == 7.0) and torch.all(out_buf[-pad:] == 7.0)
    assert torch.all(lse_buf[:pad] == 7.0) and torch.all(lse_buf[-pad:] == 7.0)
    assert torch.all(ws_buf[:pad] == 7.0) and torch.all(ws_buf[pad + need // 4:] == 7.0)
    ref, rl = reference(w)
    assert_close(host_bf16(out.view(w.B, w.Hq, w.D)), lse.view(w.B, w.Hq).cpu().numpy().astype(
        np.float64), ref, rl, "canary")


def test_null_lse_and_side_stream():
    import torch
    w = wl.make_problem(2, 32, 8, 128, 2048, seed=13)
    d = OnDevice(w)
    ref, _ = reference(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, lse, _ = d.run(4, with_lse=False, stream=s)
    s.synchronize()
    got = host_bf16(out)
    assert np.max(np.abs(got - ref)) <= 1e-2


def test_error_codes_with_real_pointers():
    import torch
    w = wl.make_problem(1, 8, 8, 128, 512, seed=14)
    d = OnDevice(w)
    out = torch.empty((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    need = fd.fd_workspace_bytes(1, 8, 128, 8)
    ws = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    assert fd.fd_decode(d.problem(), d.q, d.k, d.v, None, None, w.scale, 8, out, None, ws,
                        need - 256, None) == fd.FD_ERR_WORKSPACE
    assert fd.fd_decode(d.problem(), d.q, d.k, d.v, None, None, w.scale, 8, out, None, None,
                        0, None) == fd.FD_ERR_WORKSPACE
    assert fd.fd_decode(d.problem(), d.q, d.k, d.v, None, None, -1.0, 1, out, None, None, 0,
                        None) == fd.FD_ERR_INVALID_ARGUMENT
    assert fd.fd_check_device_error() == fd.FD_OK


def test_planner_on_device_matches_pure_planner():
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for L in (512, 16384, 65536):
        assert fd.fd_plan(1, 64, 8, 128, L, 0) == fd.fd_plan_sm(sms, 1, 64, 8, 128, L, 0)
        for kv in (fd.FD_KV_BF16, fd.FD_KV_FP8_E4M3):
            prob = fd.make_problem(1, 64, 8, 128, L, kv_dtype=kv)
            assert fd.fd_plan_problem(0, prob) == fd.fd_plan_problem(sms, prob)
