"""The seeded input generator: published SplitMix64 vectors, distribution,
bf16 rounding, thread-count independence and the workload recipes."""
import math

import numpy as np
import pytest

from split_kv_decode_attn_b200 import workloads as wl


def test_splitmix64_published_vectors():
    # SplitMix64 reference outputs for seed 1234567 and seed 0.
    assert [int(x) for x in wl.u64(1234567, 5)] == [
        6457827717110365317, 3203168211198807973, 9817491932198370423,
        4593380528125082431, 16408922859458223821]
    assert int(wl.u64(0, 1)[0]) == 0xE220A8397B1DCDAF


def test_counter_based_random_access():
    a = wl.u64(99, 100)
    b = wl.u64(99, 10, offset=90)
    assert np.array_equal(a[90:], b)


def test_normal_moments_and_bf16_rounding():
    z = wl.normal_f64(7, 1 << 20)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    bits = wl.normal_bf16(7, (1 << 20,))
    # bf16 = RNE of the fp32 rounding of the fp64 draw
    assert np.array_equal(bits, wl.f64_to_bf16_bits(z))
    back = wl.bf16_bits_to_f64(bits)
    assert np.max(np.abs(back - z) / np.maximum(np.abs(z), 1e-30)) <= 2.0 ** -8 * 1.0001


def test_thread_count_does_not_change_values():
    a = wl.normal_bf16(5, (300001,), nthreads=1)
    b = wl.normal_bf16(5, (300001,), nthreads=7)
    assert np.array_equal(a, b)


def test_f64_to_bf16_ties_to_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1.0078125: rounds to even (1.0)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0])
    got = wl.f64_to_bf16_bits(x)
    assert list(got) == [0x3F80, 0x3F82, 0xC020, 0x0000]


def test_permutation_and_positions():
    p = wl.permutation(11, 1000)
    assert sorted(p.tolist()) == list(range(1000))
    assert not np.array_equal(p, np.arange(1000))
    pos = wl.distinct_positions(12, 64, 262144)
    assert len(set(pos.tolist())) == 64 and pos.min() >= 0 and pos.max() < 262144


def test_uniform_int_range():
    x = wl.uniform_int(13, 10000, 1024, 32768)
    assert x.min() >= 1024 and x.max() <= 32768
    assert abs(x.mean() - (1024 + 32768) / 2) < 300


def test_small_problem_layouts():
    w = wl.make_problem(2, 8, 2, 64, 96, seed=3, seqlens=[96, 50], nan_pad=True)
    assert w.k.shape == (2, 2, 96, 64) and w.q.shape == (2, 8, 64)
    assert np.all(w.k[1, :, 50:] == wl.BF16_NAN) and np.all(w.v[1, :, 50:] == wl.BF16_NAN)
    assert not np.any(w.k[0] == wl.BF16_NAN)
    assert w.kv_bytes() == (96 + 50) * 2 * 64 * 4
    p = wl.make_problem(2, 8, 2, 64, 96, seed=3, block_size=16)
    assert p.k.shape == (12, 2, 16, 64) and p.block_table.shape == (2, 6)
    assert sorted(p.block_table.ravel().tolist()) == list(range(12))
    k, v = p.logical_kv(1, 1)
    pages = p.block_table[1]
    assert np.array_equal(k[16:32], p.k[pages[1], 1])


def test_dominant_key_recipe():
    w = wl.make_problem(1, 8, 2, 128, 1024, seed=5)
    pos = wl.plant_dominant_keys(w, 8, seed=5)
    q0 = wl.bf16_bits_to_f64(w.q[0, 4])  # group of KV head 1 starts at query head 4
    kk = wl.bf16_bits_to_f64(w.k[0, 1, pos[0]])
    s = float(np.float32(w.scale)) * float(q0 @ kk)
    assert s == pytest.approx(4 * np.linalg.norm(q0), rel=1e-2)


def test_config_recipes_are_the_stated_shapes():
    c1 = wl.config(1)
    assert (c1.B, c1.Hq, c1.Hkv, c1.D, c1.max_len) == (1, 8, 8, 64, 512)
    assert c1.scale == np.float32(1 / math.sqrt(64))
    c2 = wl.config(2, L=512)
    assert (c2.B, c2.Hq, c2.Hkv, c2.D, c2.max_len) == (1, 64, 8, 128, 512)
    sl = wl.uniform_int(wl.stream_seed(wl.CONFIG_SEED_BASE + 3, wl.STREAM_SEQLENS),
                        32, 1024, 32768)
    assert sl.min() >= 1024 and sl.max() <= 32768 and len(sl) == 32


def test_token_major_layouts():
    n = wl.make_problem(2, 8, 2, 64, 96, seed=3, seqlens=[96, 50], nan_pad=True, layout="NHD")
    assert n.k.shape == (2, 96, 2, 64) and n.kv_layout == 1
    assert np.all(n.k[1, 50:] == wl.BF16_NAN) and not np.any(n.k[0] == wl.BF16_NAN)
    k, v = n.logical_kv(1, 1)
    assert k.shape == (50, 64) and np.array_equal(k, n.k[1, :50, 1])
    p = wl.make_problem(2, 8, 2, 64, 96, seed=3, block_size=16, layout="NHD")
    assert p.k.shape == (12, 16, 2, 64)
    k, v = p.logical_kv(0, 1)
    assert np.array_equal(k[16:32], p.k[p.block_table[0, 1], :, 1])


def test_e4m3_codec_against_the_format_definition():
    """OCP FP8 E4M3: bias 7, 3 mantissa bits, subnormals m * 2^-9, S.1111.111
    is NaN, largest finite 448."""
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0,
             0xFE: -448.0}
    for c, val in table.items():
        assert wl.e4m3_bits_to_f64(np.array([c]))[0] == val
    assert np.isnan(wl.e4m3_bits_to_f64(np.array([0x7F, 0xFF]))).all()
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    back = wl.f64_to_e4m3_bits(wl.e4m3_bits_to_f64(finite))
    assert np.array_equal(back, finite)
    # nearest, ties to even, saturation
    x = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -11, 500.0, -1e9, 0.3])
    assert list(wl.f64_to_e4m3_bits(x)) == [0x38, 0x3A, 0x00, 0x01, 0x7E, 0xFE, 0x2A]


def test_fp8_workload_recipe():
    w = wl.make_problem(2, 8, 2, 128, 64, seed=4, seqlens=[64, 10], nan_pad=True, kv_dtype="fp8")
    assert w.k.dtype == np.uint8 and w.kv_dtype_code == 1 and w.k_scale == 1 / 32
    assert np.all(w.k[1, :, 10:] == 0x7F)
    k, _ = w.logical_kv_f64(0, 1)
    assert np.isfinite(k).all() and 0.8 < np.std(k) < 1.2
    assert w.kv_bytes() == (64 + 10) * 2 * 128 * 2
