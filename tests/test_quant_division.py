"""Host check of the quantizer kernel's division by 6.

The NVFP4 quantizer computes its block scale from (amax * gs) / 6 rounded to float32 and then to
E4M3.  The kernel does not divide: it corrects the product by the rounded reciprocal,
z = RN(1/6), q0 = RN(p z), r = p - 6 q0 (exact with an FMA), q1 = RN(q0 + r z)
(Markstein's method for a divisor known in advance; Brisebarre, Muller and Raina, IEEE Trans.
Computers 53(8), 2004).  This test proves in exact integer arithmetic that q1 == RN(p / 6) for all
2^23 float32 significands, which covers every p whose quotient is a normal float32 (scaling p by
a power of two scales every step exactly).  It also checks that the uncorrected product q0 is
wrong for many of them, so that a dropped correction step would not pass.
"""

import numpy as np

RECIP6_BITS = 0x3E2AAAAB          # float32 RN(1/6) = 0x1.555556p-3, the kernel's constant


def _rne(num, den, bits=24):
    """num/den (positive int64 arrays, quotient >= 2^(bits-1)) rounded to nearest even at `bits`
    significant bits; returns the rounded value as an integer in the units of num/den."""
    q = num // den
    e = np.floor(np.log2(q.astype(np.float64))).astype(np.int64) - (bits - 1)
    e = np.where((q >> np.maximum(e + bits - 1, 0)) == 0, e - 1, e)      # guard the float log2
    e = np.where((q >> np.maximum(e + bits, 0)) != 0, e + 1, e)
    assert (e >= 0).all()
    d = den << e
    m = num // d
    rem = num - m * d
    m = m + ((2 * rem > d) | ((2 * rem == d) & (m % 2 == 1)))
    over = (m >> bits) != 0
    m = np.where(over, m >> 1, m)
    e = np.where(over, e + 1, e)
    return m << e


def test_recip6_constant_is_rounded_reciprocal():
    z = np.array([RECIP6_BITS], dtype=np.uint32).view(np.float32)[0]
    assert z == np.float32(1.0) / np.float32(6.0)
    assert float(z) == float.fromhex("0x1.555556p-3")
    # Z * 2^-26 with Z the nearest integer to 2^26 / 6
    assert float(z) * 2 ** 26 == round(2 ** 26 / 6)


def test_fma_corrected_quotient_is_correctly_rounded_for_all_significands():
    P = np.arange(1 << 23, 1 << 24, dtype=np.int64)     # p = P * 2^-23 in [1, 2)
    Z = round(2 ** 26 / 6)                               # z = Z * 2^-26
    q0 = _rne(P * Z, np.full_like(P, 1 << 23))           # RN(p z), units of 2^-26
    r = 8 * P - 6 * q0                                   # p - 6 q0, exact, units of 2^-26
    assert np.abs(r).max() <= 9
    q1 = _rne((q0 << 26) + r * Z, np.ones_like(P))       # RN(q0 + r z), units of 2^-52
    want = _rne(P << 29, np.full_like(P, 6))             # RN(p / 6), units of 2^-52
    np.testing.assert_array_equal(q1, want)
    # the correction step matters: the product alone misses about a third of the cases
    assert ((q0 << 26) != want).sum() > (1 << 23) // 4


def test_rne_helper_against_float32_division():
    """The integer rounding helper agrees with numpy's float32 division on a sample (so the
    exhaustive check above compares against the right definition of RN(p / 6))."""
    rng = np.random.default_rng(7)
    P = rng.integers(1 << 23, 1 << 24, size=4096, dtype=np.int64)
    want = (P.astype(np.float32) * np.float32(2.0 ** -23)) / np.float32(6.0)
    got = _rne(P << 29, np.full_like(P, 6)).astype(np.float64) * 2.0 ** -52
    np.testing.assert_array_equal(got.astype(np.float32), want)
