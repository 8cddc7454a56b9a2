"""The INT4 attention's accumulator rescale, emulated exactly on the CPU.

When a row's running max moves, its int32 P.V accumulator acc (16 x the
integer sum of w * v) is scaled by alpha = 2^(m_old - m_new) in (0, 1] in
place: t = fl(float(acc) * alpha + 1.5 * 2^23) (one FMA), acc' = bits(t) -
bits(1.5 * 2^23).  Rows with 2^15 <= l < 2^21 take acc * alpha / 64 the same
way and multiply back by 64; rows with l >= 2^21 use / 4096.  The claims: the
short path gives exactly rne(acc * alpha) for |acc| < 2^22; the /64 path is
within 64 units for |acc| < 2^28; the /4096 path is within 4096 units over
the accumulator's whole range (|acc| <= 112 l <= 1680 N for N <= 2^19 tokens,
the longest sequence the host accepts).  The kernel keeps the accumulator as
MB + acc (MB = bits of 1.5 * 2^23): short-path rows rescale MB + acc with one
FMA (within one unit, below), the others subtract MB first.

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


def rescale_long(acc, alpha, div=64):
    sc = (alpha * np.float32(1.0 / div)).astype(np.float32)   # exact: a power of two
    t = fma32(acc.astype(np.float32), sc, MAGIC32)
    # the kernel forms bits(t) * div - bits(MAGIC) * div in uint32 arithmetic
    u = (t.view(np.uint32).astype(np.uint64) * np.uint64(div)
         + (np.uint64(1 << 32) - np.uint64(int(MAGIC_BITS) * div % (1 << 32)))) % np.uint64(1 << 32)
    return u.astype(np.uint32).view(np.int32).astype(np.int64)


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


def test_huge_path_error_bound_over_int32():
    rng = np.random.default_rng(14)
    top = 112 * 15 * (1 << 19)          # largest |acc| of the longest accepted sequence
    acc = rng.integers(-top, top + 1, 400000, dtype=np.int64)
    acc[:2] = [top, -top]
    a = alphas(rng, acc.size)
    got = rescale_long(acc, a, 4096)
    exact = acc.astype(np.float64) * a.astype(np.float64)
    assert np.max(np.abs(got - exact)) <= 4096.0


def test_accumulator_bound_at_the_longest_sequence():
    # 112 = |16 * 7| (widened V code), 15 = largest P weight: the worst row of
    # the longest accepted sequence, on top of the offset MB, still fits int32
    n_max = 1 << 19
    assert int(MAGIC_BITS) + 112 * 15 * n_max < (1 << 31)
    assert int(MAGIC_BITS) - 112 * 15 * n_max > -(1 << 31)
    # the tier thresholds: the exact path needs 112 l < 2^22 for l < 2^15,
    # the /64 path 112 l < 2^28 for l < 2^21
    assert 112 * (1 << 15) < (1 << 22)
    assert 112 * (1 << 21) < (1 << 28)


def rescale_offset(stored, alpha):
    """The accumulator kept as MB + a (MB = bits of 1.5 * 2^23): for |a| < 2^22
    the stored word read as a float is 1.5 * 2^23 + a, and one FMA with
    beta = fl(1.5 * 2^23 (1 - alpha)) gives the stored word of the rescaled a."""
    f = stored.astype(np.uint32).view(np.float32)
    beta = fma32(np.full(alpha.shape, -MAGIC32, np.float32), alpha, MAGIC32)
    t = (f.astype(np.float64) * alpha.astype(np.float64) + beta.astype(np.float64)).astype(np.float32)
    return t.view(np.uint32).astype(np.int64)


def test_offset_accumulator_path_within_one_unit():
    rng = np.random.default_rng(15)
    a = rng.integers(-(1 << 22) + 1, 1 << 22, 400000, dtype=np.int64)
    a[:3] = [(1 << 22) - 1, -(1 << 22) + 1, 0]
    al = alphas(rng, a.size)
    stored = a + int(MAGIC_BITS)
    got = rescale_offset(stored, al) - int(MAGIC_BITS)
    exact = a.astype(np.float64) * al.astype(np.float64)
    assert np.max(np.abs(got - exact)) <= 1.0
