"""CPU check of the arithmetic behind the rotated quantiser's row divisor.

The kernel forms fl(amax / q) (q = 127 for INT8, 7 for INT4) as
fl(amax * hi + fl(amax * lo)), with hi = fl32(1 / q) and lo = fl32(1 / q - hi)
(one fp32 product and one fma). Here that composition is evaluated exactly
with numpy (the product amax * lo is exact in float64, and so is the sum
amax * hi + fl32(amax * lo): together they span at most 52 bits), rounded once
to fp32 at each step as the fma and the product do, and compared with the
IEEE fp32 quotient for every fp32 significand of a binade. Scaling by a power
of two leaves both sides' rounding unchanged while every intermediate stays
a normal number; the lowest binade the fast path takes (amax >= 2^-103, where
fl32(amax * lo) is subnormal) is checked on its own. The kernel's
own output is compared the same way on the GPU
(test_gpu_parity.py::test_row_divisor_is_the_ieee_quotient).
"""
import numpy as np
import pytest

HI_LO = {
    127: (float.fromhex("0x1.020408p-7"), float.fromhex("0x1.020408p-35")),
    7: (float.fromhex("0x1.24924ap-3"), float.fromhex("-0x1.b6db6ep-28")),
}


def all_significands(exponent: int) -> np.ndarray:
    bits = (np.uint32(127 + exponent) << np.uint32(23)) | np.arange(1 << 23, dtype=np.uint32)
    return bits.view(np.float32)


def two_word_quotient(a: np.ndarray, q: int) -> np.ndarray:
    hi, lo = HI_LO[q]
    a64 = a.astype(np.float64)
    p = (a64 * lo).astype(np.float32)  # exact product, one rounding
    return (a64 * hi + p.astype(np.float64)).astype(np.float32)  # exact sum, one rounding


@pytest.mark.parametrize("q", [127, 7])
def test_constants_are_the_two_word_reciprocal(q):
    from fractions import Fraction

    hi, lo = HI_LO[q]
    assert np.float32(hi) == hi and np.float32(lo) == lo
    exact = Fraction(1, q)
    # hi is the nearest fp32 to 1/q, lo the nearest fp32 to the remainder
    for x, target in ((hi, exact), (lo, exact - Fraction(hi))):
        f = np.float32(x)
        for nb in (np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))):
            assert abs(Fraction(float(f)) - target) <= abs(Fraction(float(nb)) - target)
    rel = abs(exact - Fraction(hi) - Fraction(lo)) / exact
    assert rel < Fraction(1, 2 ** 50)


@pytest.mark.parametrize("q", [127, 7])
@pytest.mark.parametrize("exponent", [-103, 0])
def test_two_word_quotient_is_the_ieee_quotient(q, exponent):
    a_all = all_significands(exponent)
    for c in range(0, a_all.size, 1 << 20):  # chunks keep the temporaries small
        a = a_all[c:c + (1 << 20)]
        expect = a / np.float32(q)  # IEEE fp32 division, correctly rounded
        got = two_word_quotient(a, q)
        bad = np.flatnonzero(got.view(np.uint32) != expect.view(np.uint32))
        assert bad.size == 0, (q, exponent, a[bad[:5]])


def test_a_single_product_is_not_enough():
    """Negative control: fl(amax * hi) alone misrounds some significands, so
    the test above would notice a dropped lo term."""
    a = all_significands(0)[: 1 << 20]
    hi, _ = HI_LO[127]
    one = (a.astype(np.float64) * hi).astype(np.float32)
    assert np.count_nonzero(one.view(np.uint32) != (a / np.float32(127)).view(np.uint32)) > 0
