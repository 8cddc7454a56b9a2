"""The prologue kernels' division-free INT4 code, emulated exactly on the CPU.

The kernels do not divide per element: with r = RN(1/s) they form
t = fl(v r + 1.5 * 2^23) (one FMA; its low mantissa bits are rne(v r)) and
e = fl(v r - rne(v r)) (a second FMA), and fall back to the IEEE quotient
rne(fl(v / s)) when |e| > 0.49999.  The claim is that the result always
equals clamp(rne(fl(v / s)), -7, 7) for |v| <= amax and s = fl(amax / 7).

float32 products are exact in float64 (24 + 24 bits), so an FMA is the
float64 sum rounded once to float32; numpy's float32 division is IEEE.  The
samples include values placed a few ulps around every half-integer quotient,
where the two roundings could differ.
"""
import numpy as np

MAGIC = np.float64(12582912.0)   # 1.5 * 2^23


def fma32(a, b, c):
    """fl32(a * b + c) with one rounding (a, b float32; the product is exact in float64)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c).astype(np.float32)


def code_ieee(v, s):
    q = np.rint(np.float32(v) / np.float32(s))      # rne of the IEEE float32 quotient
    return np.clip(q, -7, 7).astype(np.int32)


def code_reciprocal(v, s):
    r = (np.float32(1.0) / s).astype(np.float32)
    t = fma32(v, r, MAGIC)
    k = (t.astype(np.float64) - MAGIC)               # exact: t is on the integer grid
    e = fma32(v, r, -k)
    near_tie = np.abs(e) > np.float32(0.49999)
    fast = k.astype(np.int32)
    return np.where(near_tie, code_ieee(v, s), fast), near_tie


def block(rng, n, amax):
    v = (rng.uniform(-1.0, 1.0, n) * amax).astype(np.float32)
    v[0], v[1] = np.float32(amax), np.float32(-amax)
    return v


def test_reciprocal_code_equals_ieee_code_on_random_blocks():
    rng = np.random.default_rng(7)
    for amax in rng.lognormal(0.0, 3.0, 200).astype(np.float32):
        s = (amax / np.float32(7.0)).astype(np.float32)
        v = block(rng, 4096, amax)
        got, tie = code_reciprocal(v, s)
        assert np.array_equal(got, code_ieee(v, s))
        assert got.min() >= -7 and got.max() <= 7
        assert tie.mean() < 1e-3                     # the IEEE fallback is rare on ordinary values


def test_reciprocal_code_equals_ieee_code_next_to_every_tie():
    """v a few ulps around (k + 1/2) s for every k: the only places where
    rne(v r) and rne(fl(v / s)) may part; the fallback must catch them."""
    rng = np.random.default_rng(8)
    fallbacks = 0
    total = 0
    parted = 0
    for amax in rng.lognormal(0.0, 2.0, 300).astype(np.float32):
        s = (amax / np.float32(7.0)).astype(np.float32)
        ties = ((np.arange(-7, 7) + 0.5).astype(np.float64) * np.float64(s)).astype(np.float32)
        v = []
        for tv in ties:
            x = tv
            for _ in range(12):                      # walk 12 ulps down and up from the tie
                x = np.nextafter(x, np.float32(-np.inf))
            for _ in range(25):
                v.append(x)
                x = np.nextafter(x, np.float32(np.inf))
        v = np.array(v, np.float32)
        v = v[np.abs(v) <= amax]
        got, tie = code_reciprocal(v, s)
        want = code_ieee(v, s)
        assert np.array_equal(got, want), amax
        fallbacks += int(tie.sum())
        total += v.size
        r = (np.float32(1.0) / s).astype(np.float32)
        fast = (fma32(v, r, MAGIC).astype(np.float64) - MAGIC).astype(np.int32)
        parted += int((fast != want).sum())
    assert fallbacks == total                        # within 12 ulps of a tie, always the IEEE quotient
    assert parted > 0                                # and without the fallback some codes would differ


def test_fast_path_needs_no_clamp_and_its_low_nibble_is_the_code():
    rng = np.random.default_rng(9)
    amax = np.float32(3.25)
    s = (amax / np.float32(7.0)).astype(np.float32)
    v = block(rng, 100000, amax)
    r = (np.float32(1.0) / s).astype(np.float32)
    t = fma32(v, r, MAGIC)
    k = (t.astype(np.float64) - MAGIC).astype(np.int64)
    assert k.min() >= -7 and k.max() <= 7            # |v r| < 7.5: no clamp
    nib = t.view(np.uint32) & 0xF                    # 0x4B400000 is a multiple of 16
    assert np.array_equal(nib, (k & 0xF).astype(np.uint32))
