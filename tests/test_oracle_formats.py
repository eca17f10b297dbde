"""Pins of the oracle's element decoders and its single fp64 -> bf16 rounding step.

Each check ties the oracle to something other than itself: the format definitions' fixed points
(largest finite value, smallest subnormal, NaN codes, value count), an independent library decoder
(torch's float8 type), the library's fp32 -> bf16 conversion on fp32-exact inputs, hand-derived
double-rounding cases, and the exact rational rounding of ``oracle.brute``.
"""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from nvfp4_grouped_gemm_indices_b200 import workloads as W


def test_e4m3_table_fixed_points():
    v = oracle.dec_e4m3(np.arange(256, dtype=np.uint8))
    nan_codes = [c for c in range(256) if math.isnan(v[c])]
    assert nan_codes == [0x7F, 0xFF]
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert v[0x01] == 2.0 ** -9          # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert v[0x08] == 2.0 ** -6          # smallest normal
    assert v[0x38] == 1.0                # exponent field 7 = bias
    assert v[0x00] == 0.0 and math.copysign(1.0, v[0x80]) == -1.0
    pos = v[0x01:0x7F]
    assert len(pos) == 126 and np.all(np.diff(pos) > 0)
    for c in range(0x80):
        if c != 0x7F:
            assert v[c | 0x80] == -v[c]


def test_e4m3_matches_library_decoder():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.dec_e4m3(codes)
    both_nan = np.isnan(lib) & np.isnan(ours)
    assert np.all(both_nan | (lib == ours))


def test_e2m1_table():
    v = oracle.dec_e2m1(np.arange(16, dtype=np.uint8))
    assert list(v[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(v[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert math.copysign(1.0, v[8]) == -1.0
    assert np.all(np.isfinite(v))


def test_e2m1_matches_library_decoder_when_available():
    try:
        packed = torch.arange(256, dtype=torch.uint8).view(torch.float4_e2m1fn_x2)
        # no CPU conversion exists in some builds; skip in that case
        lib = packed.to(torch.float32)
    except Exception:
        pytest.skip("library has no float4 -> float conversion")
    lib = lib.numpy().astype(np.float64).reshape(-1)
    raw = np.arange(256, dtype=np.uint8)
    ours = np.stack([oracle.dec_e2m1(raw & 0xF), oracle.dec_e2m1(raw >> 4)], axis=-1).reshape(-1)
    assert lib.size in (256, 512)
    if lib.size == 512:
        assert np.all(lib == ours)


def test_quantiser_roundtrip_against_decoder():
    """encode(decode(c)) == c for every finite E4M3 and every E2M1 code: ties the generator's
    encoders and the oracle's decoders to each other (they share no code)."""
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.dec_e4m3(codes)
    fin = ~np.isnan(dec)
    assert np.array_equal(W.e4m3_encode(dec[fin].astype(np.float32)), codes[fin])
    nib = np.arange(16, dtype=np.uint8)
    assert np.array_equal(W.e2m1_encode(oracle.dec_e2m1(nib).astype(np.float32)), nib)


def _bf16_bits_via_fp32(x32):
    t = torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().astype(np.uint16)


def test_bf16_rounding_matches_library_on_fp32_exact_values():
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    # add exact ties: bf16 grid points plus half an ulp
    ties = (rng.integers(0, 2 ** 16, size=2000, dtype=np.uint32) << 16) | 0x8000
    tie_vals = ties.view(np.float32)
    tie_vals = tie_vals[np.isfinite(tie_vals)]
    x = np.concatenate([x, tie_vals]).astype(np.float32)
    ours = oracle.bf16_from_f64(x.astype(np.float64))
    lib = _bf16_bits_via_fp32(x)
    assert np.array_equal(ours, lib)


@pytest.mark.parametrize("x,expected", [
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),   # just above a tie: rounds up (fp32 detour would give 0x3F80)
    (1.0 + 2.0 ** -8, 0x3F80),                # exact tie -> even
    (1.0 + 3 * 2.0 ** -8, 0x3F82),            # exact tie -> even (up)
    (1.0 + 2.0 ** -8 - 2.0 ** -45, 0x3F80),   # just below a tie
    (-(1.0 + 2.0 ** -8 + 2.0 ** -40), 0xBF81),
    (2.0 ** 128 - 2.0 ** 119, 0x7F80),        # tie above the largest finite (odd mantissa) -> Inf
    (2.0 ** 128 - 2.0 ** 119 - 2.0 ** 80, 0x7F7F),
    (1e300, 0x7F80), (-1e300, 0xFF80),
    (2.0 ** -133, 0x0001),                    # smallest subnormal
    (2.0 ** -134, 0x0000),                    # tie to even (zero)
    (3 * 2.0 ** -134, 0x0002),                # tie to even (2)
    (2.0 ** -134 + 2.0 ** -160, 0x0001),
    (2.0 ** -126 - 2.0 ** -134, 0x0080),      # tie rounds up into the smallest normal
    (0.0, 0x0000), (-0.0, 0x8000),
    (float("inf"), 0x7F80), (float("-inf"), 0xFF80),
])
def test_bf16_rounding_hand_cases(x, expected):
    assert int(oracle.bf16_from_f64([x])[0]) == expected
    if math.isfinite(x) and x != 0.0:  # a rational has no signed zero
        from fractions import Fraction
        assert brute.bf16_round(Fraction(x)) == expected


def test_bf16_nan():
    assert int(oracle.bf16_from_f64([float("nan")])[0]) & 0x7FFF == 0x7FC0


def test_bf16_rounding_matches_exact_rational_on_random_doubles():
    from fractions import Fraction
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(3000) * np.exp2(rng.integers(-140, 130, 3000)),
        rng.standard_normal(500),
    ])
    ours = oracle.bf16_from_f64(xs)
    for x, o in zip(xs, ours):
        assert brute.bf16_round(Fraction(float(x))) == int(o), x
