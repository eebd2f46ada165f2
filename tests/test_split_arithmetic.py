"""Exactness of the operand splits the apply products read (no GPU).

The CUDA kernels split the roots once per refresh: XL into three bf16 planes
(each the nearest bf16 to what the previous planes leave) and XR into the
3xTF32 hi part (round to 11 significant bits) and its fp32 remainder.  The
design relies on both being exact: the planes sum to XL, and hi + lo = XR.
These tests restate the two rounding rules in numpy on the bit patterns and
check the sums exactly over values of every magnitude a root can take, so a
wrong claim in either rule would fail here before any GPU run.
"""
import numpy as np


def bf16_nearest(x32):
    """Nearest bf16 (ties to even) of finite float32 values, as float32."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32)


def tf32_hi(x32):
    """The hi part of the 3xTF32 split: round half away at bit 13, keep 19 bits."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x1000) & 0xFFFFE000).astype(np.uint32).view(np.float32)


def sample(seed):
    rng = np.random.default_rng(seed)
    mant = rng.standard_normal(200_000)
    expo = rng.integers(-100, 100, size=mant.size)
    x = (mant * 2.0 ** expo).astype(np.float32)
    return x[np.isfinite(x) & (x != 0)]


def test_three_bf16_planes_sum_to_the_value_exactly():
    x = sample(1)
    p0 = bf16_nearest(x)
    r1 = (x - p0).astype(np.float32)
    p1 = bf16_nearest(r1)
    r2 = (r1 - p1).astype(np.float32)
    p2 = bf16_nearest(r2)
    # each remainder is exact in fp32, and the last one needs no rounding
    assert np.array_equal(x.astype(np.float64) - p0.astype(np.float64), r1.astype(np.float64))
    assert np.array_equal(r1.astype(np.float64) - p1.astype(np.float64), r2.astype(np.float64))
    assert np.array_equal(p2, r2)
    total = p0.astype(np.float64) + p1.astype(np.float64) + p2.astype(np.float64)
    assert np.array_equal(total, x.astype(np.float64))
    # every plane is a bf16 value (its low 16 bits are zero)
    for p in (p0, p1, p2):
        assert not np.any(p.view(np.uint32) & 0xFFFF)


def test_two_planes_would_not_be_enough():
    """Two planes keep 16 significant bits: the third is needed for fp32 roots."""
    x = sample(2)
    p0 = bf16_nearest(x)
    p1 = bf16_nearest((x - p0).astype(np.float32))
    two = p0.astype(np.float64) + p1.astype(np.float64)
    assert np.mean(two != x.astype(np.float64)) > 0.9


def test_tf32_hi_and_remainder_sum_exactly():
    x = sample(3)
    hi = tf32_hi(x)
    lo = (x - hi).astype(np.float32)
    assert np.array_equal(hi.astype(np.float64) + lo.astype(np.float64), x.astype(np.float64))
    assert not np.any(hi.view(np.uint32) & 0x1FFF)          # 10 stored mantissa bits
    assert np.all(np.abs(lo) <= np.abs(x) * 2.0 ** -11)     # the remainder is small
