"""The INT4 attention's accumulator rescale, emulated exactly on the CPU.

When a row's running max moves, its int32 P.V accumulator acc (16 x the
integer sum of w * v) is scaled by alpha = 2^(m_old - m_new) in (0, 1] in
place: t = fl(float(acc) * alpha + 1.5 * 2^23) (one FMA), acc' = bits(t) -
bits(1.5 * 2^23).  Rows with l >= 2^15 take acc * alpha / 64 the same way and
multiply back by 64.  The claims: the short path gives exactly rne(acc * alpha)
for |acc| < 2^22; the long path is within 64 units for |acc| < 2^28.

float32 products are exact in float64, so the FMA is the float64 sum rounded
once to float32; float32(int) is round-to-nearest like cvt.rn.f32.s32.
"""
import numpy as np

MAGIC32 = np.float32(12582912.0)
MAGIC_BITS = np.int64(0x4B400000)


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)


def rescale_short(acc, alpha):
    t = fma32(acc.astype(np.float32), alpha, MAGIC32)
    return t.view(np.int32).astype(np.int64) - MAGIC_BITS


def rescale_long(acc, alpha):
    sc = (alpha * np.float32(0.015625)).astype(np.float32)   # exact: a power of two
    t = fma32(acc.astype(np.float32), sc, MAGIC32)
    return (t.view(np.int32).astype(np.int64) - MAGIC_BITS) * 64


def alphas(rng, n):
    a = np.exp2(-rng.exponential(2.0, n)).astype(np.float32)
    a[:4] = [1.0, 0.5, np.float32(2.0 ** -20), np.nextafter(np.float32(1.0), np.float32(0.0))]
    return a


def test_short_path_is_the_nearest_integer():
    rng = np.random.default_rng(11)
    acc = rng.integers(-(1 << 22) + 1, 1 << 22, 400000, dtype=np.int64)
    acc[:3] = [(1 << 22) - 1, -(1 << 22) + 1, 0]
    a = alphas(rng, acc.size)
    got = rescale_short(acc, a)
    exact = acc.astype(np.float64) * a.astype(np.float64)    # exact in float64 (22 + 24 bits)
    want = np.rint(exact).astype(np.int64)                   # round half to even
    assert np.array_equal(got, want)


def test_long_path_error_bound():
    rng = np.random.default_rng(12)
    acc = rng.integers(-(1 << 28) + 1, 1 << 28, 400000, dtype=np.int64)
    a = alphas(rng, acc.size)
    got = rescale_long(acc, a)
    exact = acc.astype(np.float64) * a.astype(np.float64)
    assert np.max(np.abs(got - exact)) <= 64.0


def test_short_path_breaks_past_its_range():
    """Past 2^22 the short path no longer rounds to the nearest integer, which
    is why rows with a large normaliser take the long one."""
    rng = np.random.default_rng(13)
    acc = rng.integers(1 << 24, 1 << 27, 100000, dtype=np.int64)
    a = np.full(acc.size, np.float32(0.999), np.float32)
    got = rescale_short(acc, a)
    want = np.rint(acc.astype(np.float64) * np.float64(a[0])).astype(np.int64)
    assert not np.array_equal(got, want)
