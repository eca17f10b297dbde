"""Exact rational brute force for tiny cases -- TEST INFRASTRUCTURE ONLY.

Pure Python with ``fractions.Fraction``: every decoded element, product, block sum, scale product
and the final sum are exact rationals; the single bf16 rounding is done on the exact value.  It is
written independently of ``bsg_oracle.c`` (different decoding route, different rounding route) so
that the C oracle can be pinned against it bit for bit on shapes small enough for pure-Python loops.
"""
from fractions import Fraction
import math
import struct


def e4m3_value(code):
    """Exact value of an E4M3 (FN) code, or None for NaN."""
    code &= 0xFF
    if code & 0x7F == 0x7F:
        return None
    neg = code >= 0x80
    mag = code & 0x7F
    exp_field = mag // 8
    frac_field = mag % 8
    if exp_field == 0:
        v = Fraction(frac_field, 512)
    else:
        v = Fraction(8 + frac_field, 8) * (Fraction(2) ** (exp_field - 7))
    return -v if neg else v


def e2m1_value(nib):
    nib &= 0xF
    neg = nib >= 8
    mag = nib % 8
    exp_field = mag // 2
    frac_field = mag % 2
    if exp_field == 0:
        v = Fraction(frac_field, 2)
    else:
        v = Fraction(2 + frac_field, 2) * (Fraction(2) ** (exp_field - 1))
    return -v if neg else v


def f32_value(x):
    """Exact rational value of a (finite) fp32 number."""
    return Fraction(struct.unpack("<f", struct.pack("<f", float(x)))[0])


def bf16_round(v):
    """Exact rational -> bf16 bit pattern, round to nearest, ties to even mantissa."""
    if v == 0:
        return 0
    neg = v < 0
    a = -v if neg else v
    # find e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 7)
    q = a / ulp
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * ulp
    sign = 0x8000 if neg else 0
    if r >= Fraction(2) ** 128:
        return sign | 0x7F80
    if r < Fraction(2) ** -126:
        return sign | int(r / Fraction(2) ** -133)
    e2 = r.numerator.bit_length() - r.denominator.bit_length()
    if Fraction(2) ** e2 > r:
        e2 -= 1
    mant = int((r / Fraction(2) ** e2 - 1) * 128)
    return sign | ((e2 + 127) << 7) | mant


def fp8_grouped(A, B, a_scale, b_scale, m_indices, M, N, K, G):
    """Returns {(m, n): bf16 bits} for routed rows only."""
    KB = K // 128
    out = {}
    for m in range(M):
        g = 0 if m_indices is None else int(m_indices[m])
        if g < 0 or g >= G:
            continue
        for n in range(N):
            total = Fraction(0)
            for kb in range(KB):
                part = Fraction(0)
                for k in range(kb * 128, kb * 128 + 128):
                    part += e4m3_value(int(A[m][k])) * e4m3_value(int(B[g][n][k]))
                total += f32_value(a_scale[m][kb]) * f32_value(b_scale[g][n // 128][kb]) * part
            out[(m, n)] = bf16_round(total)
    return out


def nvfp4(A, B, sfa, sfb, alpha, m_indices, M, N, K, G):
    """A, B packed (two E2M1 per byte, low nibble first).  Returns {(m, n): bf16 bits}."""
    def elem(row, k):
        byte = int(row[k // 2])
        return e2m1_value(byte & 0xF if k % 2 == 0 else byte >> 4)

    out = {}
    for m in range(M):
        g = 0 if m_indices is None else int(m_indices[m])
        if g < 0 or g >= G:
            continue
        for n in range(N):
            total = Fraction(0)
            for j in range(K // 16):
                blk = Fraction(0)
                for k in range(j * 16, j * 16 + 16):
                    blk += elem(A[m], k) * elem(B[g][n], k)
                total += e4m3_value(int(sfa[m][j])) * e4m3_value(int(sfb[g][n][j])) * blk
            out[(m, n)] = bf16_round(f32_value(alpha[g]) * total)
    return out
