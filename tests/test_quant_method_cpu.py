"""CPU checks of the arithmetic the activation-quantiser kernels use in place of divisions, written
out in exact rational arithmetic (no GPU, no oracle):

* amax / 448 and amax / 6 for every non-negative bf16 amax: the product with the rounded reciprocal
  of the divisor, corrected once by its exact remainder, is the correctly rounded fp32 quotient;
* the two bracketing products x * r(1 -+ 2^-21) fall on either side of the correctly rounded quotient
  when r is a hardware reciprocal within 1 ulp of 1/d refined by one Newton step, over random operands.
"""
from fractions import Fraction

import numpy as np


def rn32(x: Fraction) -> np.float32:
    """Round a rational to the nearest fp32 (ties to even), subnormals included."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    e = max(e, -126)
    q = x / Fraction(2) ** (e - 23)
    n = q.numerator // q.denominator
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(sign * float(Fraction(n) * Fraction(2) ** (e - 23)))


def F(v):
    return Fraction(float(v))


def test_corrected_product_is_the_correctly_rounded_quotient_for_every_bf16():
    a_all = (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    for d in (448.0, 6.0):
        c = np.float32(1.0) / np.float32(d)
        for a in a_all:
            s0 = np.float32(a * c)                               # RN(a * c)
            e = rn32(F(a) - F(s0) * Fraction(int(d)))            # fma(-s0, d, a)
            s = rn32(F(e) * F(c) + F(s0))                        # fma(e, c, s0)
            assert s.view(np.uint32) == np.float32(a / np.float32(d)).view(np.uint32), (d, a)


def test_bracketing_products_enclose_the_quotient():
    rng = np.random.default_rng(3)
    lo_f, hi_f = np.float32(1 - 2.0 ** -21), np.float32(1 + 2.0 ** -21)
    for _ in range(3000):
        d = np.float32(rng.uniform(1e-3, 1e3))
        x = np.float32(rng.choice([-1, 1]) * rng.uniform(0, 448) * d)
        q = rn32(F(x) / F(d))
        r_rn = np.float32(1) / d
        for r0 in (r_rn, np.nextafter(r_rn, np.float32(0)), np.nextafter(r_rn, np.float32(1e9))):  # within 1 ulp
            e = rn32(1 - F(d) * F(r0))                  # fma(-d, r0, 1)
            r = rn32(F(r0) * F(e) + F(r0))              # fma(r0, e, r0)
            q_lo = rn32(F(x) * F(rn32(F(r) * F(lo_f))))
            q_hi = rn32(F(x) * F(rn32(F(r) * F(hi_f))))
            lo, hi = (q_lo, q_hi) if x >= 0 else (q_hi, q_lo)
            assert lo <= q <= hi


def test_bracket_codes_differ_by_at_most_one_without_borrow():
    """The kernels take their flags from (packed codes of x r(1 + 2^-21)) - (packed codes of
    x r(1 - 2^-21)): this needs every element's two codes to be equal or adjacent, the larger one from
    the larger product, with the same sign bit -- checked here with the input generators' encoders on
    products spread over every binade of both formats (near cell boundaries included)."""
    from nvfp4_grouped_gemm_indices_b200 import workloads as W

    rng = np.random.default_rng(11)
    lo_f, hi_f = np.float32(1 - 2.0 ** -21), np.float32(1 + 2.0 ** -21)
    # magnitudes across the whole code range, plus exact midpoints and their fp32 neighbours
    mags = np.concatenate([
        np.float32(2.0) ** rng.uniform(-12, 9.2, 20000).astype(np.float32),
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 2.0 ** -10, 1.0625, 464.0, 0.0], np.float32),
    ]).astype(np.float32)
    mags = np.concatenate([mags, np.nextafter(mags, np.float32(0)), np.nextafter(mags, np.float32(1e9))])
    q = (mags * rng.choice(np.array([-1, 1], np.float32), mags.size)).astype(np.float32)
    q_lo = (q * lo_f).astype(np.float32)
    q_hi = (q * hi_f).astype(np.float32)
    for enc, sign_bit in ((W.e4m3_encode, 0x80), (W.e2m1_encode, 0x8)):
        c_lo = enc(q_lo).astype(np.int32)
        c_hi = enc(q_hi).astype(np.int32)
        assert np.array_equal(c_lo & sign_bit, c_hi & sign_bit)           # same sign bit
        d = c_hi - c_lo                                                   # magnitude codes: no borrow
        assert d.min() >= 0 and d.max() <= 1
        assert d.sum() > 0                                                # the boundary cases occur
