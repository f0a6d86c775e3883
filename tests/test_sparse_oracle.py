"""Pins of the sparse-decode oracle (oracle/sparse.py): the low-bit codes, the
scan's error bound, the top-delta rule's special cases, and the reduction to
the dense oracle when every block is kept."""
import importlib.util
import os

import numpy as np
import pytest

import oracle
from split_kv_decode_attn_b200 import workloads as wl


def _sparse_oracle():
    """oracle.sparse, or the copy named by FD_SPARSE_ORACLE (the mutant tests
    run these pins against copies with one planted slip)."""
    path = os.environ.get("FD_SPARSE_ORACLE")
    if not path:
        from oracle import sparse as module
        return module
    spec = importlib.util.spec_from_file_location("sparse_under_test", path)
    module = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(module)
    return module


sparse = _sparse_oracle()

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def exact_kept(q, k8, sk, scale, delta, num_splits, seqlens=None):
    return sparse.select_blocks_exact(q, k8, sk, scale, delta, num_splits, seqlens)[0]


# The rule's pins run on both forms of the selection: the fp32 product order
# the library uses, and the fp64 definition.
SELECTORS = {"fp32": lambda *a, **kw: sparse.select_blocks(*a, **kw), "fp64": exact_kept}


def problem(B=3, Hq=8, Hkv=2, D=64, L=300, seed=1, lens=(300, 130, 1)):
    return wl.make_problem(B, Hq, Hkv, D, L, seed=seed, seqlens=list(lens), nan_pad=True)


def f32(bits):
    return wl.bf16_bits_to_f64(bits).astype(np.float32)


def test_key_codes_round_to_the_block_scale():
    w = problem()
    k8, sk = sparse.quantize_keys(w.k, w.seqlens)
    B, Hkv, L, D = w.k.shape
    assert k8.dtype == np.int8 and k8.shape == w.k.shape and sk.shape == (B, Hkv, 5)
    assert np.abs(k8.astype(np.int32)).max() <= 127
    for b in range(B):
        n = int(w.seqlens[b])
        for h in range(Hkv):
            for blk in range(5):
                r0, r1 = blk * 64, min(L, blk * 64 + 64)
                rows = np.arange(r0, r1)
                valid = rows < n
                codes = k8[b, h, r0:r1].astype(np.float64)
                assert np.all(codes[~valid] == 0)          # padding (NaN here) takes no part
                if not valid.any():
                    assert sk[b, h, blk] == 1.0
                    continue
                kv = f32(w.k[b, h, rows[valid]]).astype(np.float64)
                s = float(sk[b, h, blk])
                assert s == np.float32(np.abs(kv).max() / np.float32(127))
                assert np.abs(codes[valid]).max() == 127    # the largest entry maps to 127
                # half a step, plus the fp32 rounding of the scale and of the quotient
                assert np.all(np.abs(kv - s * codes[valid]) <= s / 2 * (1 + 1e-5))


def test_zero_block_and_query_codes():
    k = np.zeros((1, 1, 64, 64), np.uint16)
    k8, sk = sparse.quantize_keys(k)
    assert np.all(k8 == 0) and sk[0, 0, 0] == 1.0
    q8, sq = sparse.quantize_query(np.zeros((2, 64), np.uint16))
    assert np.all(q8 == 0) and np.all(sq == 1.0)
    w = problem()
    q8, sq = sparse.quantize_query(w.q)
    qf = f32(w.q).astype(np.float64)
    assert np.all(np.abs(q8).max(axis=-1) == 127)
    assert np.all(np.abs(qf - sq[..., None] * q8) <= sq[..., None] / 2 * (1 + 1e-5))


def test_scan_logits_stay_within_the_quantisation_bound():
    """|s~ - s| <= scale * sum_d (|q_d| dk/2 + |k_d| dq/2 + dq dk/4) plus fp32
    rounding, with dq, dk the query and block scales."""
    w = problem(B=1, Hq=4, Hkv=1, D=128, L=256, seed=3, lens=(256,))
    k8, sk = sparse.quantize_keys(w.k)
    q8, sq = sparse.quantize_query(w.q)
    qf = f32(w.q[0]).astype(np.float64)
    kf = f32(w.k[0, 0]).astype(np.float64)
    for g in range(4):
        for j in range(256):
            dk = float(sk[0, 0, j // 64])
            approx = float(np.float32(np.float32(np.float32(w.scale) * sq[0, g]) * np.float32(dk))
                           * np.float32(int(q8[0, g].astype(np.int64) @ k8[0, 0, j].astype(np.int64))))
            exact = w.scale * qf[g] @ kf[j]
            bound = w.scale * (np.abs(qf[g]) @ np.full(128, dk / 2) + np.abs(kf[j]).sum() * sq[0, g] / 2
                               + 128 * sq[0, g] * dk / 4)
            assert abs(approx - exact) <= bound + 1e-5 * abs(exact) + 1e-6


def test_infinite_delta_keeps_everything_and_equals_dense_attention():
    w = problem(B=3, Hq=8, Hkv=2, D=64, L=300, lens=(300, 130, 0))
    for S in (1, 3):
        out, lse, kept = sparse.sparse_decode(w.q, w.k, w.v, w.scale, np.inf, S, w.seqlens)
        ref, rl = oracle.decode(w.q, w.k, w.v, w.scale, seqlens=w.seqlens)
        assert np.array_equal(out, ref) and np.array_equal(lse, rl)
        for b, n in enumerate(w.seqlens):
            nb = -(-int(n) // 64)
            assert kept[b, :, :nb].all() and not kept[b, :, nb:].any()


@pytest.mark.parametrize("form", sorted(SELECTORS))
def test_one_dominant_block_selects_alone(form):
    """The selection alone, in both forms: a key aligned with every query
    head of the group, far above the rest, is the only block kept at
    delta = 0 with one split."""
    w = problem(B=1, Hq=4, Hkv=1, D=128, L=1024, seed=5, lens=(1024,))
    qf = f32(w.q[0]).astype(np.float64)
    key = qf.sum(axis=0)
    k = w.k.copy()
    k[0, 0, 700] = wl.f64_to_bf16_bits(24.0 * key / np.linalg.norm(key))
    k8, sk = sparse.quantize_keys(k)
    kept = SELECTORS[form](w.q, k8, sk, w.scale, 0.0, 1)
    assert kept[0, 0].tolist() == [i == 700 // 64 for i in range(16)]


def test_one_dominant_block_is_all_that_a_zero_delta_keeps():
    """A key aligned with every query head of the group, far above the rest:
    with one split and delta = 0 only its block survives, and the output is
    close to that key's value row."""
    w = problem(B=1, Hq=4, Hkv=1, D=128, L=1024, seed=5, lens=(1024,))
    qf = f32(w.q[0]).astype(np.float64)
    key = qf.sum(axis=0)
    key = 24.0 * key / np.linalg.norm(key)
    k = w.k.copy()
    k[0, 0, 700] = wl.f64_to_bf16_bits(key)
    out, lse, kept = sparse.sparse_decode(w.q, k, w.v, w.scale, 0.0, 1)
    assert kept[0, 0].tolist() == [i == 700 // 64 for i in range(16)]
    v700 = wl.bf16_bits_to_f64(w.v[0, 0, 700])
    assert np.abs(out[0] - v700).max() < 0.05


@pytest.mark.parametrize("form", sorted(SELECTORS))
def test_more_delta_keeps_more_and_each_split_keeps_its_best_block(form):
    select = SELECTORS[form]
    w = wl.make_problem(2, 8, 2, 128, 2048, seed=9, seqlens=[2048, 1500])
    k8, sk = sparse.quantize_keys(w.k, w.seqlens)
    prev = None
    for delta in (0.0, 0.5, 1.0, 2.0, 4.0, np.inf):
        kept = select(w.q, k8, sk, w.scale, delta, 4, w.seqlens)
        if prev is not None:
            assert np.all(kept >= prev)                    # monotone in delta
        prev = kept
    kept0 = select(w.q, k8, sk, w.scale, 0.0, 4, w.seqlens)
    for b in range(2):
        nb = -(-int(w.seqlens[b]) // 64)
        for h in range(2):
            for s0, s1 in sparse.split_blocks(2048, 4):
                if s0 < nb:
                    assert kept0[b, h, s0:min(nb, s1)].any()
            assert not kept0[b, h, nb:].any()


@pytest.mark.parametrize("form", sorted(SELECTORS))
def test_kept_blocks_are_the_union_over_the_heads_of_a_group(form):
    """Two query heads of one group, each with its own dominant key in a
    different block: with one split and delta = 0 exactly those two blocks
    survive, one chosen by each head (a rule that looked at one head only, or
    at the sum over heads, would keep one)."""
    w = problem(B=1, Hq=2, Hkv=1, D=128, L=1024, seed=21, lens=(1024,))
    qf = f32(w.q[0]).astype(np.float64)
    k = w.k.copy()
    for g, pos in ((0, 130), (1, 900)):
        key = 24.0 * qf[g] / np.linalg.norm(qf[g])
        k[0, 0, pos] = wl.f64_to_bf16_bits(key)
    k8, sk = sparse.quantize_keys(k)
    kept = SELECTORS[form](w.q, k8, sk, w.scale, 0.0, 1)
    assert kept[0, 0].tolist() == [i in (130 // 64, 900 // 64) for i in range(16)]
    # each head alone keeps only its own block
    for g, pos in ((0, 130), (1, 900)):
        one = SELECTORS[form](w.q[:, g:g + 1], k8, sk, w.scale, 0.0, 1)
        assert one[0, 0].tolist() == [i == pos // 64 for i in range(16)]


def test_split_blocks_follow_the_dense_cut():
    """T = ceil(max_len / 64) blocks into min(S, T) splits of floor(s T / S)
    boundaries: sizes differ by at most one block."""
    assert sparse.split_blocks(2048, 4) == [(0, 8), (8, 16), (16, 24), (24, 32)]
    assert sparse.split_blocks(1000, 3) == [(0, 5), (5, 10), (10, 16)]   # T = 16
    assert sparse.split_blocks(65, 2) == [(0, 1), (1, 2)]
    assert sparse.split_blocks(10, 16) == [(0, 1)]
    assert sparse.split_blocks(0, 4) == [(0, 0)]
    assert sparse.split_blocks(262144, 16) == [(256 * s, 256 * (s + 1)) for s in range(16)]
    # 256 blocks in 18 splits: floor(8 * 256 / 18) = 113, floor(9 * 256 / 18) = 128
    sizes = [b - a for a, b in sparse.split_blocks(16384, 18)]
    assert sum(sizes) == 256 and set(sizes) == {14, 15}
    assert [i for i, n in enumerate(sizes) if n == 15] == [4, 8, 13, 17]


@pytest.mark.parametrize("form", sorted(SELECTORS))
def test_top_delta_applies_per_split_of_the_balanced_cut(form):
    """Block maxima that fall with the block index and delta = 0: each split
    keeps exactly its first block, so the kept blocks are the splits' first
    blocks, 0, 5 and 10 for 16 blocks in 3 splits (equal chunks of
    ceil(16 / 3) = 6 blocks would keep 0, 6 and 12)."""
    w = problem(B=1, Hq=1, Hkv=1, D=128, L=1024, seed=23, lens=(1024,))
    qf = f32(w.q[0, 0]).astype(np.float64)
    k = w.k.copy()
    for blk in range(16):
        key = (20.0 - blk) * np.sqrt(128.0) * qf / np.linalg.norm(qf)
        k[0, 0, 64 * blk + 3] = wl.f64_to_bf16_bits(key)
    k8, sk = sparse.quantize_keys(k)
    select = SELECTORS[form]
    kept = select(w.q, k8, sk, w.scale, 0.0, 3)
    assert np.flatnonzero(kept[0, 0]).tolist() == [0, 5, 10]
    kept = select(w.q, k8, sk, w.scale, 0.0, 16)
    assert kept[0, 0].all()                       # one block per split
    kept = select(w.q, k8, sk, w.scale, 0.0, 1)
    assert np.flatnonzero(kept[0, 0]).tolist() == [0]


def test_exact_block_maxima_by_brute_force():
    """block_maxima_exact against the logits written out token by token with
    Python integers and fractions-free fp64 products, on a tiny ragged case."""
    w = problem(B=2, Hq=4, Hkv=2, D=64, L=150, seed=31, lens=(150, 70))
    k8, sk = sparse.quantize_keys(w.k, w.seqlens)
    q8, sq = sparse.quantize_query(w.q)
    maxima = sparse.block_maxima_exact(w.q, k8, sk, w.scale, w.seqlens)
    for b, n in enumerate((150, 70)):
        for h in range(2):
            bm = maxima[(b, h)]
            assert bm.shape == (-(-n // 64), 2)
            for blk in range(bm.shape[0]):
                for g in range(2):
                    best = -np.inf
                    for j in range(blk * 64, min(n, blk * 64 + 64)):
                        dot = sum(int(x) * int(y) for x, y in zip(q8[b, 2 * h + g], k8[b, h, j]))
                        best = max(best, float(np.float32(w.scale)) * float(sq[b, 2 * h + g])
                                   * float(sk[b, h, blk]) * dot)
                    assert bm[blk, g] == pytest.approx(best, rel=1e-15, abs=0)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_fp32_rule_agrees_with_the_exact_scan_outside_the_rounding_margin(G):
    """The fp32 product order the library follows and the fp64 definition of
    the scan keep the same blocks wherever the decision lies farther from its
    threshold than fp32 rounding can move it (select_blocks_exact's
    'certain'); the blocks inside that margin are counted and must be rare."""
    lens = [0, 1, 65, 700, 2000, 3333]
    w = wl.make_problem(len(lens), 2 * G, 2, 128, 3333, seed=410 + G, seqlens=lens,
                        nan_pad=True)
    k8, sk = sparse.quantize_keys(w.k, w.seqlens)
    inside = total = 0
    for S in (1, 3, 7):
        for delta in (0.0, 2.0, 6.0):
            kept32 = sparse.select_blocks(w.q, k8, sk, w.scale, delta, S, w.seqlens)
            kept64, certain = sparse.select_blocks_exact(w.q, k8, sk, w.scale, delta, S,
                                                         w.seqlens)
            for b, n in enumerate(lens):
                nb = -(-n // 64)
                c = certain[b, :, :nb]
                assert np.array_equal(kept32[b, :, :nb][c], kept64[b, :, :nb][c])
                inside += int((~c).sum())
                total += c.size
    print(f"G={G}: {inside} of {total} block decisions inside the fp32 rounding margin")
    assert inside <= max(2, total // 1000)
