"""GPU parity of the sparse decode: fd_quantize_keys and fd_decode_sparse
(through the C ABI) against the oracle in oracle/sparse.py.

The kept-block masks are checked twice:
- against the scan's definition in fp64 (select_blocks_exact), on every block
  whose decision lies outside the fp32 rounding margin; the blocks inside it
  are counted and reported;
- bit for bit against the oracle's fp32 form of the rule, which takes the
  library's product order.
The outputs are compared with the fp64 attention over the kept blocks at the
usual tolerances."""
import numpy as np
import pytest

import split_kv_decode_attn_b200 as fd
from oracle import sparse
from split_kv_decode_attn_b200 import workloads as wl

from fdtest import OnDevice, assert_close, free_device, host_bf16, reference, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_device):
    yield
    free_device()


def torch():
    import torch as _t
    return _t


def n_blocks(w):
    return -(-w.max_len // 64)


def quantize_on_gpu(d: OnDevice):
    t = torch()
    w = d.w
    k8 = t.empty(w.k.shape, dtype=t.int8, device="cuda")
    sk = t.empty((w.B, w.Hkv, n_blocks(w)), dtype=t.float32, device="cuda")
    assert fd.fd_quantize_keys(d.problem(), d.k, d.seqlens, k8, sk) == fd.FD_OK
    return k8, sk


def run_sparse(d: OnDevice, k8, sk, delta: float, S: int):
    t = torch()
    w = d.w
    out = t.empty((w.B, w.Hq, w.D), dtype=t.bfloat16, device="cuda")
    lse = t.empty((w.B, w.Hq), dtype=t.float32, device="cuda")
    kept = t.full((w.B, w.Hkv, n_blocks(w)), 255, dtype=t.uint8, device="cuda")
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.D, S)
    ws = t.empty(max(nbytes, 4) // 4, dtype=t.float32, device="cuda")
    st = fd.fd_decode_sparse(d.problem(), d.q, d.k, d.v, k8, sk, d.seqlens, w.scale, delta, S,
                             out, lse, kept, ws, nbytes)
    assert st == fd.FD_OK, fd.fd_status_string(st)
    t.cuda.synchronize()
    assert fd.fd_check_device_error() == fd.FD_OK
    return host_bf16(out), lse.cpu().numpy().astype(np.float64), kept.cpu().numpy()


def check_kept(w, kept_gpu, kept_ref):
    for b in range(w.B):
        nb = -(-int(w.lengths()[b]) // 64)
        assert np.array_equal(kept_gpu[b, :, :nb].astype(bool), kept_ref[b, :, :nb]), b
        assert np.all(kept_gpu[b, :, nb:] == 255)     # past the length: not written


def check_kept_exact(w, kept_gpu, k8, sk, delta, S, what=""):
    """The GPU's kept blocks equal the fp64 definition's on every block whose
    decision no fp32 rounding can flip; returns (inside the margin, total)."""
    kept64, certain = sparse.select_blocks_exact(w.q, k8, sk, w.scale, delta, S, w.seqlens)
    inside = total = 0
    for b in range(w.B):
        nb = -(-int(w.lengths()[b]) // 64)
        c = certain[b, :, :nb]
        got = kept_gpu[b, :, :nb].astype(bool)
        assert np.array_equal(got[c], kept64[b, :, :nb][c]), f"{what} sequence {b}"
        inside += int((~c).sum())
        total += c.size
    print(f"{what}: {inside} of {total} block decisions inside the fp32 rounding margin")
    return inside, total


@pytest.mark.parametrize("D", [64, 128])
def test_quantize_keys_bit_exact(D):
    w = wl.make_problem(3, 8, 4, D, 1000, seed=400 + D, seqlens=[1000, 130, 0], nan_pad=True)
    d = OnDevice(w)
    k8, sk = quantize_on_gpu(d)
    ref8, refs = sparse.quantize_keys(w.k, w.seqlens)
    assert np.array_equal(sk.cpu().numpy(), refs)
    assert np.array_equal(k8.cpu().numpy(), ref8)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_sparse_decode_matches_oracle(G):
    D = 128
    Hkv = 2
    lens = [0, 1, 65, 700, 2000, 3333]
    w = wl.make_problem(len(lens), G * Hkv, Hkv, D, 3333, seed=410 + G, seqlens=lens,
                        nan_pad=True)
    d = OnDevice(w)
    k8, sk = quantize_on_gpu(d)
    ref8, refs = sparse.quantize_keys(w.k, w.seqlens)
    inside = total = 0
    for S in (1, 3, 7):
        for delta in (0.0, 2.0, 6.0):
            got, gl, kept = run_sparse(d, k8, sk, delta, S)
            ref, rl, kref = sparse.sparse_decode(w.q, w.k, w.v, w.scale, delta, S, w.seqlens,
                                                 k8=ref8, sk=refs)
            i, t = check_kept_exact(w, kept, ref8, refs, delta, S, f"G={G} S={S} delta={delta}")
            inside += i
            total += t
            check_kept(w, kept, kref)
            assert_close(got, gl, ref, rl, f"sparse G={G} S={S} delta={delta}")
    assert inside <= max(2, total // 1000)


def test_infinite_delta_is_dense_decode_bit_for_bit():
    w = wl.make_problem(3, 32, 8, 128, 5000, seed=430, seqlens=[5000, 4097, 1])
    d = OnDevice(w)
    k8, sk = quantize_on_gpu(d)
    for S in (1, 5):
        got, gl, kept = run_sparse(d, k8, sk, float("inf"), S)
        dense, dl, _ = run_gpu(d, S)
        assert np.array_equal(got, dense) and np.array_equal(gl, dl)
        for b in range(3):
            nb = -(-int(w.seqlens[b]) // 64)
            assert np.all(kept[b, :, :nb] == 1)


def test_sparse_decode_is_deterministic():
    w = wl.make_problem(2, 32, 8, 128, 8192, seed=440, seqlens=[8192, 6000])
    d = OnDevice(w)
    k8, sk = quantize_on_gpu(d)
    a, la, ka = run_sparse(d, k8, sk, 3.0, 4)
    for _ in range(3):
        b, lb, kb = run_sparse(d, k8, sk, 3.0, 4)
        assert np.array_equal(a, b) and np.array_equal(la, lb) and np.array_equal(ka, kb)


def test_peaked_long_context():
    """The peaked workload (B=1, Hq=32, Hkv=8, L=256K, 64 keys that dominate
    the first query head of each group) in the planner's split count: the kept
    masks match the oracle's for every KV head and the outputs match on two
    sampled KV heads.  The other heads of a group attend broadly, so the
    top-delta rule keeps every block: the rule adapts to the distribution."""
    check_peaked(wl.config(5), 8.0, 1.0, 1.0)


def test_group_peaked_long_context_keeps_few_blocks():
    """Same shape, with the 64 keys aligned with the whole query group: now
    every head is peaked and the rule keeps a few per cent of the blocks."""
    check_peaked(wl.peaked_group(), 8.0, 0.0, 0.1)


def check_peaked(w, delta, share_lo, share_hi):
    d = OnDevice(w)
    S = fd.fd_plan_problem(0, d.problem(), None)
    k8, sk = quantize_on_gpu(d)
    got, gl, kept = run_sparse(d, k8, sk, delta, S)
    # the oracle's own codes, one KV head at a time (memory), then the GPU's
    # codes must equal them bit for bit
    parts = [sparse.quantize_keys(w.k[:, h:h + 1], None) for h in range(w.Hkv)]
    ref8 = np.concatenate([p[0] for p in parts], axis=1)
    refs = np.concatenate([p[1] for p in parts], axis=1)
    assert np.array_equal(k8.cpu().numpy(), ref8) and np.array_equal(sk.cpu().numpy(), refs)
    inside, total = check_kept_exact(w, kept, ref8, refs, delta, S, f"{w.name} S={S}")
    assert inside <= max(2, total // 1000)
    kref = sparse.select_blocks(w.q, ref8, refs, w.scale, delta, S)
    check_kept(w, kept, kref)
    ref, rl, _ = sparse.sparse_decode(w.q, w.k, w.v, w.scale, delta, S, groups=[(0, 0), (0, 5)],
                                      k8=ref8, sk=refs)
    e = assert_close(got, gl, ref, rl, f"peaked sparse S={S}")
    share = kept.astype(bool).mean()
    dense_ref, dense_l = reference(w, groups=[(0, 0)])
    gap = float(np.nanmax(np.abs(ref - dense_ref)[0, :4]))
    print(f"{w.name} sparse S={S} delta={delta} kept {100 * share:.2f} % of blocks, "
          f"errors {e}, sparse-vs-dense max|dO| {gap:.3e}")
    assert share_lo <= share <= share_hi


def test_sparse_decode_replays_from_a_cuda_graph():
    t = torch()
    w = wl.make_problem(2, 32, 8, 128, 4096, seed=450, seqlens=[4096, 3000])
    d = OnDevice(w)
    k8, sk = quantize_on_gpu(d)
    eager, el, ek = run_sparse(d, k8, sk, 2.0, 3)
    out = t.empty((w.B, w.Hq, w.D), dtype=t.bfloat16, device="cuda")
    lse = t.empty((w.B, w.Hq), dtype=t.float32, device="cuda")
    kept = t.full((w.B, w.Hkv, n_blocks(w)), 255, dtype=t.uint8, device="cuda")
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.D, 3)
    ws = t.empty(nbytes // 4, dtype=t.float32, device="cuda")
    s = t.cuda.Stream()
    g = t.cuda.CUDAGraph()
    with t.cuda.graph(g, stream=s):
        st = fd.fd_decode_sparse(d.problem(), d.q, d.k, d.v, k8, sk, d.seqlens, w.scale, 2.0, 3,
                                 out, lse, kept, ws, nbytes, s.cuda_stream)
    assert st == fd.FD_OK
    for _ in range(3):
        g.replay()
    t.cuda.synchronize()
    assert fd.fd_check_device_error() == fd.FD_OK
    assert np.array_equal(host_bf16(out), eager)
    assert np.array_equal(lse.cpu().numpy().astype(np.float64), el)
    assert np.array_equal(kept.cpu().numpy(), ek)
