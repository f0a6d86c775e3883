"""The e4m3 splits that the tcgen05 fp8 path relies on, checked on the CPU with
the workloads' e4m3 codec (round to nearest even, saturating; pinned in
tests/test_workloads.py):

- a bf16 value x of a head whose largest magnitude is f 2^e (f in [0.5, 1))
  is scaled by sigma = 2^(8 - e), so |x sigma| < 256, and split into two codes
  x sigma = x1 + x2 / 16 with x1 = e4m3(x sigma), x2 = e4m3(16 (x sigma - x1));
  the split is exact wherever the residual is a normal e4m3 value, and
  otherwise off by at most half the subnormal spacing, 2^-10 / 16;
- a softmax weight p in (0, 256] split into three codes p1 + p2 / 16 + p3 / 256
  (each residual scaled and rounded the same way) keeps about 12 significant
  bits: a relative error of at most 2^-12 from 2^-2 up."""
import numpy as np

from split_kv_decode_attn_b200 import workloads as wl


def e4m3(x):
    return wl.e4m3_bits_to_f64(wl.f64_to_e4m3_bits(x))


def all_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]          # drop inf and NaN patterns
    return wl.bf16_bits_to_f64(bits)


def test_bf16_splits_into_two_codes():
    x = all_finite_bf16()
    x = x[x != 0]
    for e in range(-20, 21):
        # a head whose largest magnitude is in [2^(e-1), 2^e)
        xs = x[np.abs(x) < 2.0 ** e]
        xs = xs[np.abs(xs) >= 2.0 ** (e - 12)]     # twelve binades of dynamic range
        sigma = 2.0 ** (8 - e)
        y = xs * sigma
        assert np.all(np.abs(y) < 256)
        x1 = e4m3(y)
        r = (y - x1) * 16.0
        x2 = e4m3(r)
        err = np.abs(x1 + x2 / 16.0 - y)
        normal = np.abs(r) >= 2.0 ** -6
        assert np.all(err[normal] == 0.0), e
        assert np.all(err <= 2.0 ** -10 / 16.0), e


def test_weights_keep_twelve_bits_in_three_codes():
    rng = np.random.default_rng(5)
    p = np.concatenate([np.exp2(rng.uniform(-12.0, 8.0, 200000)), [256.0, 1.0, 2.0 ** -2]])
    p = np.minimum(p, 256.0)
    p1 = e4m3(p)
    r1 = p - p1
    p2 = e4m3(r1 * 16.0)
    r2 = r1 - p2 / 16.0
    p3 = e4m3(r2 * 256.0)
    q = p1 + p2 / 16.0 + p3 / 256.0
    rel = np.abs(q - p) / p
    assert np.all(rel[p >= 2.0 ** -2] <= 2.0 ** -12)
    # Two codes keep only about 8 bits: the reason for the third.
    two = p1 + p2 / 16.0
    assert np.max(np.abs(two - p)[p >= 1.0] / p[p >= 1.0]) > 2.0 ** -10
