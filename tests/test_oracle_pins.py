"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

The pages define the target only in words: the combined output equals
attention over the complete cached history ("What is Flash-Decoding, and
when does it speed up LLMs?", opening paragraph and section "Why decode needs
a different schedule"), and the split form is a partial output plus a
log-sum-exp per chunk.  So the oracle is pinned to closed forms, library
routines (scipy's softmax and logsumexp), brute force on tiny inputs and
invariances of the definition.  Each pin is chosen so that a plausible slip
(a dropped scale, a missing max shift, a wrong GQA head mapping, a log in
the wrong base, a transposed operand, an off-by-one in chunking) fails it.
"""
import math

import numpy as np
import pytest
import scipy.special

import oracle
from split_kv_decode_attn_b200 import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf(x):
    return wl.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def f64(b):
    return wl.bf16_bits_to_f64(np.asarray(b))


def rnd_bf16(seed, shape, scale=1.0):
    x = wl.normal_f64(seed, int(np.prod(shape))).reshape(shape) * scale
    return bf(x)


def scipy_attention(q, k, v, scale):
    """Library softmax over logits computed with numpy: q [G,D], k/v [n,D]."""
    qd, kd, vd = f64(q), f64(k), f64(v)
    s = float(np.float32(scale)) * (qd @ kd.T)  # [G, n]
    p = scipy.special.softmax(s, axis=1)
    return p @ vd, scipy.special.logsumexp(s, axis=1)


# --- closed forms -------------------------------------------------------------

def test_single_token_returns_v0_exactly():
    q, k, v = rnd_bf16(1, (4, 64)), rnd_bf16(2, (1, 64)), rnd_bf16(3, (1, 64))
    out, lse = oracle.attend(q, k, v, 0.125)
    assert np.array_equal(out, np.repeat(f64(v), 4, axis=0))
    for g in range(4):
        dot = math.fsum(a * b for a, b in zip(f64(q[g]), f64(k[0])))
        assert lse[g] == pytest.approx(0.125 * dot, rel=1e-14, abs=1e-14)


def test_zero_query_gives_mean_of_v_and_log_n():
    n, D = 37, 16
    q = np.zeros((2, D), np.uint16)
    k, v = rnd_bf16(4, (n, D)), rnd_bf16(5, (n, D))
    out, lse = oracle.attend(q, k, v, 0.3)
    mean = np.array([math.fsum(col) / n for col in f64(v).T])
    np.testing.assert_allclose(out[0], mean, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, math.log(n), rtol=0, atol=1e-14)


def test_identical_keys_give_mean_and_shifted_lse():
    n, D = 50, 32
    q = rnd_bf16(6, (1, D))
    k = np.repeat(rnd_bf16(7, (1, D)), n, axis=0)
    v = rnd_bf16(8, (n, D))
    scale = 0.17
    out, lse = oracle.attend(q, k, v, scale)
    s = float(np.float32(scale)) * math.fsum(a * b for a, b in zip(f64(q[0]), f64(k[0])))
    mean = np.array([math.fsum(col) / n for col in f64(v).T])
    np.testing.assert_allclose(out[0], mean, atol=1e-14)
    assert lse[0] == pytest.approx(s + math.log(n), abs=1e-13)


def test_dominant_key_returns_its_value_row_within_bound():
    n, D = 200, 64
    q = rnd_bf16(9, (1, D))
    k = rnd_bf16(10, (n, D), 0.1)
    jstar = 123
    qd = f64(q[0])
    k[jstar] = bf(6.0 * qd / np.linalg.norm(qd) * math.sqrt(D))
    v = rnd_bf16(11, (n, D))
    scale = 1.0 / math.sqrt(D)
    out, _ = oracle.attend(q, k, v, scale)
    s = float(np.float32(scale)) * (f64(k) @ qd)
    delta = s[jstar] - np.max(np.delete(s, jstar))
    assert delta > 20
    vd = f64(v)
    bound = (n - 1) * math.exp(-delta) * np.max(np.abs(vd - vd[jstar]))
    assert np.max(np.abs(out[0] - vd[jstar])) <= bound + 1e-15


def test_two_tokens_textbook_sigmoid_form():
    D = 8
    q, k, v = rnd_bf16(12, (3, D)), rnd_bf16(13, (2, D)), rnd_bf16(14, (2, D))
    scale = 0.7
    out, lse = oracle.attend(q, k, v, scale)
    sc = float(np.float32(scale))
    for g in range(3):
        s0 = sc * float(f64(q[g]) @ f64(k[0]))
        s1 = sc * float(f64(q[g]) @ f64(k[1]))
        sig = 1.0 / (1.0 + math.exp(-(s0 - s1)))
        expect = sig * f64(v[0]) + (1.0 - sig) * f64(v[1])
        np.testing.assert_allclose(out[g], expect, rtol=1e-13, atol=1e-14)
        assert lse[g] == pytest.approx(float(np.logaddexp(s0, s1)), rel=1e-14)


def test_hand_worked_example():
    """q=(1,0), K rows (0,5),(1,7),(2,3), scale 1: logits 0,1,2.
    Weights are 1, e, e^2 over Z = 1+e+e^2; V rows (1,0),(0,1),(1,1)."""
    q = bf([[1.0, 0.0]])
    k = bf([[0.0, 5.0], [1.0, 7.0], [2.0, 3.0]])
    v = bf([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    out, lse = oracle.attend(q, k, v, 1.0)
    e = math.e
    Z = 1 + e + e * e
    np.testing.assert_allclose(out[0], [(1 + e * e) / Z, (e + e * e) / Z], rtol=1e-15)
    assert lse[0] == pytest.approx(math.log(Z), rel=1e-15)


@pytest.mark.parametrize("n,D", [(1, 1), (2, 3), (3, 4), (4, 2), (4, 4)])
def test_brute_force_tiny(n, D):
    """Softmax written out by hand with plain floats, no max shift."""
    G = 2
    q, k, v = rnd_bf16(100 + n, (G, D)), rnd_bf16(200 + D, (n, D)), rnd_bf16(300 + n * D, (n, D))
    scale = 0.9
    out, lse = oracle.attend(q, k, v, scale)
    qd, kd, vd = f64(q), f64(k), f64(v)
    sc = float(np.float32(scale))
    for g in range(G):
        logits = []
        for j in range(n):
            acc = 0.0
            for d in range(D):
                acc += qd[g][d] * kd[j][d]
            logits.append(sc * acc)
        ex = [math.exp(x) for x in logits]
        tot = sum(ex)
        for d in range(D):
            o = sum(ex[j] * vd[j][d] for j in range(n)) / tot
            assert out[g][d] == pytest.approx(o, rel=1e-12, abs=1e-14)
        assert lse[g] == pytest.approx(math.log(tot), rel=1e-13, abs=1e-14)


# --- library routines and the GQA mapping ------------------------------------

@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_matches_scipy_softmax(G):
    n, D = 300, 64
    q, k, v = rnd_bf16(15 + G, (G, D)), rnd_bf16(16, (n, D)), rnd_bf16(17, (n, D))
    out, lse = oracle.attend(q, k, v, 1 / 8)
    o2, l2 = scipy_attention(q, k, v, 1 / 8)
    np.testing.assert_allclose(out, o2, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, l2, rtol=1e-13)


def test_batch_decode_gqa_mapping_and_seqlens():
    """Head h reads KV head floor(h / G); sequence b reads seqlens[b] rows."""
    B, Hq, Hkv, D, L = 3, 8, 2, 32, 40
    G = Hq // Hkv
    q = rnd_bf16(20, (B, Hq, D))
    k = rnd_bf16(21, (B, Hkv, L, D))
    v = rnd_bf16(22, (B, Hkv, L, D))
    sl = np.array([40, 1, 17], np.int32)
    out, lse = oracle.decode(q, k, v, 0.2, seqlens=sl, nthreads=3)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            o2, l2 = scipy_attention(q[b, h:h + 1], k[b, kv, :sl[b]], v[b, kv, :sl[b]], 0.2)
            np.testing.assert_allclose(out[b, h], o2[0], rtol=1e-11, atol=1e-13)
            assert lse[b, h] == pytest.approx(l2[0], rel=1e-13)


def test_large_logits_do_not_overflow():
    """Logits near +-2000 need the max shift; compare with scipy logsumexp."""
    n, D = 64, 16
    q, k, v = rnd_bf16(23, (2, D), 30.0), rnd_bf16(24, (n, D), 30.0), rnd_bf16(25, (n, D))
    out, lse = oracle.attend(q, k, v, 1.0)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    o2, l2 = scipy_attention(q, k, v, 1.0)
    np.testing.assert_allclose(out, o2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, l2, rtol=1e-13)


def test_scale_is_taken_at_float32():
    q, k, v = rnd_bf16(26, (1, 8)), rnd_bf16(27, (1, 8)), rnd_bf16(28, (1, 8))
    _, lse = oracle.attend(q, k, v, 0.1)
    dot = math.fsum(a * b for a, b in zip(f64(q[0]), f64(k[0])))
    assert lse[0] == pytest.approx(float(np.float32(0.1)) * dot, rel=1e-15, abs=1e-15)
    assert abs(lse[0] - 0.1 * dot) > 1e-10 * abs(dot) or dot == 0


# --- invariances --------------------------------------------------------------

def test_duplicated_cache_keeps_output_and_adds_log2():
    n, D = 77, 32
    q, k, v = rnd_bf16(30, (3, D)), rnd_bf16(31, (n, D)), rnd_bf16(32, (n, D))
    out, lse = oracle.attend(q, k, v, 0.25)
    out2, lse2 = oracle.attend(q, np.concatenate([k, k]), np.concatenate([v, v]), 0.25)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse2, lse + math.log(2), rtol=1e-14)


def test_permuting_kv_pairs_changes_nothing():
    n, D = 91, 32
    q, k, v = rnd_bf16(33, (2, D)), rnd_bf16(34, (n, D)), rnd_bf16(35, (n, D))
    perm = wl.permutation(36, n)
    out, lse = oracle.attend(q, k, v, 0.25)
    out2, lse2 = oracle.attend(q, k[perm], v[perm], 0.25)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=1e-14)


def test_linear_in_v():
    n, D = 64, 16
    q, k, v = rnd_bf16(37, (2, D)), rnd_bf16(38, (n, D)), rnd_bf16(39, (n, D))
    out, _ = oracle.attend(q, k, v, 0.3)
    out4, _ = oracle.attend(q, k, bf(f64(v) * -4.0), 0.3)  # exact in bf16
    np.testing.assert_allclose(out4, -4.0 * out, rtol=1e-14, atol=1e-14)


def test_constant_v_rows_reproduce_the_row():
    n, D = 64, 16
    q, k = rnd_bf16(40, (2, D)), rnd_bf16(41, (n, D))
    row = rnd_bf16(42, (1, D))
    out, _ = oracle.attend(q, k, np.repeat(row, n, axis=0), 0.3)
    np.testing.assert_allclose(out, np.repeat(f64(row), 2, axis=0), rtol=1e-14, atol=1e-15)


def test_rows_past_seqlen_are_never_read():
    B, Hq, Hkv, D, L = 2, 4, 2, 16, 24
    q = rnd_bf16(43, (B, Hq, D))
    k = rnd_bf16(44, (B, Hkv, L, D))
    v = rnd_bf16(45, (B, Hkv, L, D))
    sl = np.array([5, 24], np.int32)
    k[0, :, 5:] = wl.BF16_NAN
    v[0, :, 5:] = wl.BF16_NAN
    out, lse = oracle.decode(q, k, v, 0.25, seqlens=sl)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    o2, l2 = oracle.attend(q[0, :2], k[0, 0, :5].copy(), v[0, 0, :5].copy(), 0.25)
    np.testing.assert_array_equal(out[0, :2], o2)


def test_empty_and_clamped_lengths():
    B, Hq, Hkv, D, L = 3, 2, 1, 8, 10
    q = rnd_bf16(46, (B, Hq, D))
    k = rnd_bf16(47, (B, Hkv, L, D))
    v = rnd_bf16(48, (B, Hkv, L, D))
    out, lse = oracle.decode(q, k, v, 0.5, seqlens=np.array([0, 99, -3], np.int32))
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))
    full, lfull = oracle.decode(q, k, v, 0.5)
    np.testing.assert_array_equal(out[1], full[1])
    np.testing.assert_array_equal(lse[1], lfull[1])


# --- split then combine -------------------------------------------------------

@pytest.mark.parametrize("chunk", [1, 7, 64, 255, 256, 1000])
def test_split_combine_equals_unsplit(chunk):
    n, D = 256, 64
    q, k, v = rnd_bf16(50, (4, D)), rnd_bf16(51, (n, D)), rnd_bf16(52, (n, D))
    out, lse = oracle.attend(q, k, v, 0.125)
    out2, lse2 = oracle.attend_split(q, k, v, 0.125, chunk)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13)


def test_split_partials_are_chunk_attention():
    n, D, C = 150, 32, 64
    q, k, v = rnd_bf16(53, (2, D)), rnd_bf16(54, (n, D)), rnd_bf16(55, (n, D))
    out, lse, po, pl = oracle.attend_split(q, k, v, 0.2, C, max_parts=4)
    for s, (b, e) in enumerate([(0, 64), (64, 128), (128, 150)]):
        o_s, l_s = scipy_attention(q, k[b:e], v[b:e], 0.2)
        np.testing.assert_allclose(po[:, s], o_s, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(pl[:, s], l_s, rtol=1e-13)
    assert np.all(po[:, 3] == 0) and np.all(np.isneginf(pl[:, 3]))
    # the combine is the lse-weighted mean of the normalised partials
    w = np.exp(pl[:, :3] - pl[:, :3].max(axis=1, keepdims=True))
    comb = (w[:, :, None] * po[:, :3]).sum(1) / w.sum(1, keepdims=True)
    np.testing.assert_allclose(comb, out, rtol=1e-12, atol=1e-14)


def test_split_of_empty_sequence():
    q = rnd_bf16(56, (2, 8))
    k = np.zeros((0, 8), np.uint16)
    out, lse = oracle.attend_split(q, k, k, 0.5, 16)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_f64_inputs_match_bf16_inputs_exactly():
    """The fp64 entry point runs the same arithmetic on already-widened values."""
    n, D = 123, 64
    q, k, v = rnd_bf16(60, (4, D)), rnd_bf16(61, (n, D)), rnd_bf16(62, (n, D))
    out, lse = oracle.attend(q, k, v, 0.125)
    out2, lse2 = oracle.attend_f64(f64(q), f64(k), f64(v), float(np.float32(0.125)))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_f64_inputs_against_scipy_on_non_bf16_values():
    rng = np.random.default_rng(5)
    q, k, v = rng.normal(size=(2, 16)), rng.normal(size=(40, 16)), rng.normal(size=(40, 16))
    out, lse = oracle.attend_f64(q, k, v, 0.3)
    s = 0.3 * (q @ k.T)
    np.testing.assert_allclose(out, scipy.special.softmax(s, axis=1) @ v, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=1), rtol=1e-13)
