"""Pins of the activation-quantiser oracle (the step before the GEMM) against what the formats and
the arithmetic fix, independently of the oracle's own code:

* every finite E4M3 / E2M1 code survives encode(decode(code)) bit for bit (signed zeros included);
* the midpoint between two neighbouring codes goes to the even one, a hair either side goes to
  the nearer one; magnitudes past the largest finite value saturate;
* the quantisers agree bit for bit with the input generators' vectorised implementation (numpy
  and the library's float8 type), which shares nothing with the oracle;
* on inputs built so that the correctly rounded quotient x / scale and the product x * (1 / scale)
  round to different codes, the codes are those of the quotient (one IEEE fp32 division per
  element, the quantiser as the format recipe writes it);
* each block's largest element lands on +-448 (FP8) and dequantised values sit within half a step
  of the input; a zero block gives zero scale and zero codes;
* gathering rows first equals quantising the gathered matrix (the MoE expand).
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_grouped_gemm_indices_b200 import workloads as W


def f32_to_bf16_bits(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def test_e4m3_round_trip_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    finite = (codes & 0x7F) != 0x7F
    vals = oracle.dec_e4m3(codes[finite]).astype(np.float32)
    assert np.array_equal(oracle.enc_e4m3(vals), codes[finite])


def test_e2m1_round_trip_every_code():
    codes = np.arange(16, dtype=np.uint8)
    vals = oracle.dec_e2m1(codes).astype(np.float32)
    assert np.array_equal(oracle.enc_e2m1(vals), codes)


@pytest.mark.parametrize("kind", ["e4m3", "e2m1"])
def test_midpoints_tie_to_even_and_neighbours_to_nearest(kind):
    if kind == "e4m3":
        codes = np.arange(0, 0x7F, dtype=np.uint8)        # +0 .. 448
        dec, enc = oracle.dec_e4m3, oracle.enc_e4m3
    else:
        codes = np.arange(0, 8, dtype=np.uint8)            # +0 .. 6
        dec, enc = oracle.dec_e2m1, oracle.enc_e2m1
    v = dec(codes)
    for c0, c1, a, b in zip(codes[:-1], codes[1:], v[:-1], v[1:]):
        mid = (a + b) / 2.0                                 # exact in fp32 for these formats
        even = c0 if c0 % 2 == 0 else c1
        assert enc(np.float32(mid)) == even
        assert enc(np.nextafter(np.float32(mid), np.float32(0))) == c0
        assert enc(np.nextafter(np.float32(mid), np.float32(1e9))) == c1
        assert enc(np.float32(-mid)) == (even | (0x80 if kind == "e4m3" else 0x8))


def test_saturation():
    assert oracle.enc_e4m3(np.float32(464.0)) == 0x7E      # would round to 480: clamps to 448
    assert oracle.enc_e4m3(np.float32(1e30)) == 0x7E
    assert oracle.enc_e4m3(np.float32(-1e30)) == 0xFE
    assert oracle.enc_e2m1(np.float32(100.0)) == 0x7
    assert oracle.enc_e2m1(np.float32(-6.0001)) == 0xF


def test_encoders_match_the_generators_vectorised_encoders():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-4, 0.01, 1, 30, 600)]).astype(np.float32)
    assert np.array_equal(oracle.enc_e4m3(x), W.e4m3_encode(x))
    y = (rng.standard_normal(20000) * 3).astype(np.float32)
    assert np.array_equal(oracle.enc_e2m1(y), W.e2m1_encode(y))


def test_fp8_rows_match_generator_and_pin_the_block_maximum():
    rng = np.random.default_rng(4)
    M, K = 64, 512
    xb = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * rng.uniform(0.01, 10, (M, 1)))
    x = bf16_bits_to_f32(xb)
    A, s = oracle.quant_fp8_rows(xb)
    A_ref, s_ref = W.quant_fp8_rows(x)
    assert np.array_equal(s, s_ref) and np.array_equal(A, A_ref)
    # the largest |x| of every block maps to +-448 exactly; every value dequantises within half a step
    blocks = x.reshape(M, K // 128, 128)
    arg = np.abs(blocks).argmax(axis=-1)
    top = np.take_along_axis(A.reshape(M, K // 128, 128), arg[..., None], -1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)
    dq = oracle.dec_e4m3(A).reshape(M, K // 128, 128) * s[..., None]
    q = blocks / s[..., None]
    step = np.where(np.abs(q) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(q), 1e-30))) - 3))
    # |dec(code) - x/s| <= half a step + the quotient's own rounding (2^-24 |q|, |q| < 16 steps)
    assert np.all(np.abs(dq - blocks) <= 0.5 * step * s[..., None] * (1 + 2.0 ** -19))


def test_nvfp4_rows_match_generator():
    rng = np.random.default_rng(5)
    M, K = 48, 256
    xb = f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    x = bf16_bits_to_f32(xb)
    gs = W.nvfp4_global_scale(x)
    A, sf = oracle.quant_nvfp4_rows(xb, gs)
    A_ref, sf_ref = W.quant_nvfp4(x, gs)
    assert np.array_equal(sf, sf_ref) and np.array_equal(A, A_ref)
    # the block scale covers the block: amax / (dec(s) * gs) <= 6 * (1 + 2^-3) before saturation
    amax = np.abs(x.reshape(M, K // 16, 16)).max(-1)
    denom = oracle.dec_e4m3(sf) * np.float64(gs)
    assert np.all(amax / denom <= 6.0 * (1 + 2.0 ** -3) + 1e-9)


def test_zero_blocks_give_zero_scales_and_codes():
    xb = np.zeros((2, 256), np.uint16)
    xb[1, 128:] = f32_to_bf16_bits(np.ones(128, np.float32))
    A, s = oracle.quant_fp8_rows(xb)
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 0] == 0 and s[1, 1] == np.float32(1 / 448)
    assert np.all(A[0] == 0) and np.all(A[1, :128] == 0) and np.all(A[1, 128:] == 0x7E)
    A4, sf = oracle.quant_nvfp4_rows(xb, np.float32(1.0))
    assert np.all(sf[0] == 0) and np.all(A4[0] == 0)


def test_gather_equals_quantising_the_gathered_rows():
    rng = np.random.default_rng(6)
    M_in, M, K = 40, 70, 256
    xb = f32_to_bf16_bits(rng.standard_normal((M_in, K)).astype(np.float32))
    src = rng.integers(0, M_in, M).astype(np.int32)
    src[[3, 9]] = [-1, M_in]                                  # out of range: row left untouched
    A, s = oracle.quant_fp8_rows(xb, M=M, src_rows=src)
    ok = (src >= 0) & (src < M_in)
    A_ref, s_ref = oracle.quant_fp8_rows(xb[src[ok]])
    assert np.array_equal(A[ok], A_ref) and np.array_equal(s[ok], s_ref)
    assert np.all(A[~ok] == 0xFF) and np.all(np.isnan(s[~ok]))
    A4, sf = oracle.quant_nvfp4_rows(xb, np.float32(0.01), M=M, src_rows=src)
    A4_ref, sf_ref = oracle.quant_nvfp4_rows(xb[src[ok]], np.float32(0.01))
    assert np.array_equal(A4[ok], A4_ref) and np.array_equal(sf[ok], sf_ref)
    assert np.all(A4[~ok] == 0xFF) and np.all(sf[~ok] == 0xFF)


def test_fp8_quotient_not_reciprocal_on_adversarial_inputs():
    from adversarial import fp8_rows
    xb, adv = fp8_rows(n_blocks=48, seed=8)
    assert adv.sum() >= 200
    x = bf16_bits_to_f32(xb)
    A, s = oracle.quant_fp8_rows(xb)
    blocks = x.reshape(1, -1, 128)
    sb = s[..., None]
    div = W.e4m3_encode((blocks / sb).astype(np.float32)).reshape(A.shape)        # IEEE fp32 division
    rcp = W.e4m3_encode((blocks * (np.float32(1) / sb)).astype(np.float32)).reshape(A.shape)
    assert np.array_equal(A, div)
    assert np.all(A[adv] != rcp[adv])


def test_nvfp4_quotient_not_reciprocal_on_adversarial_inputs():
    from adversarial import nvfp4_cases
    cases = nvfp4_cases(n=10, seed=9)
    assert len(cases) == 10
    for gs, xb, adv in cases:
        x = bf16_bits_to_f32(xb).reshape(-1, 16)
        A, sf = oracle.quant_nvfp4_rows(xb, gs)
        d = (oracle.dec_e4m3(sf.reshape(-1)).astype(np.float32) * np.float32(gs)).astype(np.float32)[:, None]
        div = W.pack_e2m1(W.e2m1_encode((x / d).astype(np.float32)).reshape(1, -1))
        rcp_codes = W.e2m1_encode((x * (np.float32(1) / d)).astype(np.float32)).reshape(1, -1)
        assert np.array_equal(A, div)
        assert np.all(W.unpack_e2m1(A)[adv] != rcp_codes[adv])
