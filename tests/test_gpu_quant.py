"""GPU parity of the activation quantisers (through the C ABI) against the fp32 oracle: the codes and
scales are integers / floats decided by the same IEEE fp32 steps on both sides, so they must match
bit for bit; output rows whose source row is out of range must stay untouched."""
import numpy as np
import pytest
import torch

import nvfp4_grouped_gemm_indices_b200 as bsg
from nvfp4_grouped_gemm_indices_b200 import workloads as W
import oracle

pytestmark = pytest.mark.gpu


def make_x(M, K, seed, zero_blocks=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32) * rng.uniform(1e-3, 50, (M, 1)).astype(np.float32)
    if zero_blocks and M > 2 and K >= 256:
        x[1, 128:256] = 0.0                       # a zero FP8 block / zero NVFP4 blocks
        x[2, :16] = 0.0
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t, t.view(torch.int16).numpy().view(np.uint16).copy()


def src_map(M_in, M, seed, bad=True):
    rng = np.random.default_rng(seed)
    src = rng.integers(0, M_in, M).astype(np.int32)
    if bad and M > 4:
        src[[1, M - 2]] = [-1, M_in]              # out of range: the output row is not written
    return src


@pytest.mark.parametrize("M_in,M,K,gather", [(1, 1, 128, False), (37, 37, 384, False), (300, 300, 7168, False),
                                           (64, 150, 512, True), (200, 33, 1152, True)])
def test_fp8_rows_bit_exact(M_in, M, K, gather):
    xt, xb = make_x(M_in, K, seed=M_in + K)
    src = src_map(M_in, M, seed=K) if gather else None
    A = torch.full((M, K), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((M, K // 128), -7.0, dtype=torch.float32, device="cuda")
    src_d = None if src is None else torch.from_numpy(src).cuda()
    bsg.bsg_quantize_fp8_rows(xt.cuda(), src_d, A, s, M_in, M, K)
    torch.cuda.synchronize()
    A_ref, s_ref = oracle.quant_fp8_rows(xb, M=M, src_rows=src, A=np.full((M, K), 0xAB, np.uint8),
                                         scale=np.full((M, K // 128), -7.0, np.float32))
    assert np.array_equal(A.cpu().numpy(), A_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("M_in,M,K,gather", [(1, 1, 16, False), (29, 29, 272, False), (256, 256, 4608, False),
                                           (64, 150, 512, True), (200, 33, 1040, True)])
def test_nvfp4_rows_bit_exact(M_in, M, K, gather):
    xt, xb = make_x(M_in, K, seed=3 * M_in + K)
    gs = W.nvfp4_global_scale(xt.float().numpy())
    src = src_map(M_in, M, seed=K + 1) if gather else None
    A = torch.full((M, K // 2), 0xAB, dtype=torch.uint8, device="cuda")
    sf = torch.full((M, K // 16), 0xCD, dtype=torch.uint8, device="cuda")
    gs_d = torch.tensor([gs], dtype=torch.float32, device="cuda")
    src_d = None if src is None else torch.from_numpy(src).cuda()
    bsg.bsg_quantize_nvfp4_rows(xt.cuda(), src_d, gs_d, A, sf, M_in, M, K)
    torch.cuda.synchronize()
    A_ref, sf_ref = oracle.quant_nvfp4_rows(xb, gs, M=M, src_rows=src, A=np.full((M, K // 2), 0xAB, np.uint8),
                                            sf=np.full((M, K // 16), 0xCD, np.uint8))
    assert np.array_equal(sf.cpu().numpy(), sf_ref)
    assert np.array_equal(A.cpu().numpy(), A_ref)


def test_fp8_full_size_prefill_activations():
    """The FP8 MoE prefill activations (8192 x 7168), gathered through a random expert permutation."""
    M, K = 8192, 7168
    xt, xb = make_x(M, K, seed=11, zero_blocks=False)
    src = np.random.default_rng(12).permutation(M).astype(np.int32)
    A, s = bsg.quantize_fp8_rows(xt.cuda(), torch.from_numpy(src).cuda())
    torch.cuda.synchronize()
    A_ref, s_ref = oracle.quant_fp8_rows(xb, M=M, src_rows=src)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(A.cpu().numpy(), A_ref)


def test_nvfp4_full_size_sampled_rows():
    """The NVFP4 grouped activations (65536 x 8192); every row checked on a sample of 512 rows."""
    M, K = 65536, 8192
    rng = np.random.default_rng(13)
    xt = torch.randn((M, K), dtype=torch.float32, generator=torch.Generator().manual_seed(13)).to(torch.bfloat16)
    gs = np.float32(float(xt.float().abs().max()) / (448.0 * 6.0))
    A, sf = bsg.quantize_nvfp4_rows(xt.cuda(), torch.tensor([gs], device="cuda"))
    torch.cuda.synchronize()
    rows = np.sort(rng.choice(M, 512, replace=False)).astype(np.int32)
    xb = xt[torch.from_numpy(rows).long()].view(torch.int16).numpy().view(np.uint16)
    A_ref, sf_ref = oracle.quant_nvfp4_rows(xb, gs)
    assert np.array_equal(sf.cpu().numpy()[rows], sf_ref)
    assert np.array_equal(A.cpu().numpy()[rows], A_ref)


def test_quantise_then_gemm_matches_the_oracle_chain():
    """Expand + quantise on the GPU, then the grouped FP8 GEMM on the GPU, against the oracle's
    quantiser feeding the oracle's GEMM (identical codes give identical GEMM inputs)."""
    from gpu_util import compare, routed_mask
    rng = np.random.default_rng(21)
    T, K, N, G = 300, 512, 256, 4
    xt, xb = make_x(T, K, seed=21, zero_blocks=False)
    expert = rng.integers(0, G, T)
    order = np.argsort(expert, kind="stable").astype(np.int32)   # rows grouped by expert
    m_indices = expert[order].astype(np.int32)
    w = W.make_fp8(T, N, K, G, m_indices, seed=22)               # B and b_scale of the experts
    A, s = bsg.quantize_fp8_rows(xt.cuda(), torch.from_numpy(order).cuda())
    C = torch.full((T, N), 0, dtype=torch.bfloat16, device="cuda")
    bsg.fp8_grouped_gemm(A, torch.from_numpy(w.B).cuda(), s, torch.from_numpy(w.b_scale).cuda(),
                         torch.from_numpy(m_indices).cuda(), out=C)
    torch.cuda.synchronize()
    A_ref, s_ref = oracle.quant_fp8_rows(xb, M=T, src_rows=order)
    assert np.array_equal(A.cpu().numpy(), A_ref)
    ref, _ = oracle.fp8_grouped(A_ref, w.B, s_ref, w.b_scale, m_indices, T, N, K, G)
    compare(C.view(torch.int16).cpu().numpy().view(np.uint16), ref, routed_mask(w))


def test_fp8_adversarial_quotients_bit_exact():
    """Elements whose correctly rounded quotient x / scale and product x * (1 / scale) round to
    different E4M3 codes (built in numpy by tests/adversarial.py): the kernel must give the
    quotient's code, as the oracle does."""
    from adversarial import fp8_rows
    xb, adv = fp8_rows(n_blocks=64, seed=31)
    rows = np.repeat(xb, 3, axis=0)                      # three rows: every lane position is exercised
    rows[1] = np.roll(xb[0], 128)
    rows[2] = np.roll(xb[0], 1024)
    M, K = rows.shape
    xt = torch.from_numpy(rows.view(np.int16).copy()).view(torch.bfloat16)
    A, s = bsg.quantize_fp8_rows(xt.cuda())
    torch.cuda.synchronize()
    A_ref, s_ref = oracle.quant_fp8_rows(rows)
    assert adv.sum() >= 150
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(A.cpu().numpy(), A_ref)


def test_nvfp4_adversarial_quotients_bit_exact():
    from adversarial import nvfp4_cases
    cases = nvfp4_cases(n=16, seed=32)
    assert len(cases) == 16
    for gs, xb, adv in cases:
        M, K = xb.shape
        xt = torch.from_numpy(xb.view(np.int16).copy()).view(torch.bfloat16)
        A, sf = bsg.quantize_nvfp4_rows(xt.cuda(), torch.tensor([gs], dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        A_ref, sf_ref = oracle.quant_nvfp4_rows(xb, gs)
        assert np.array_equal(sf.cpu().numpy(), sf_ref)
        assert np.array_equal(A.cpu().numpy(), A_ref), f"gs {gs!r}"


def test_tiny_scales_and_signed_zeros():
    """Blocks so small that the fp32 reciprocal of their scale overflows, and blocks of signed zeros
    (scale 0: every code is 0, the sign of a zero input included)."""
    K = 512
    rows = np.zeros((4, K), np.uint16)
    rng = np.random.default_rng(40)
    tiny = rng.integers(0x0001, 0x0080, K).astype(np.uint16) | (rng.integers(0, 2, K).astype(np.uint16) << 15)
    rows[0] = tiny                                        # bf16 subnormals: amax / 448 is an fp32 subnormal
    rows[1, :128] = 0x8000                                # -0 everywhere in block 0
    rows[1, 128:] = (rng.standard_normal(K - 128).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    rows[2, ::2] = 0x8000                                 # -0 between normal values
    rows[2, 1::2] = 0x3F80
    rows[3] = (rng.standard_normal(K).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    xt = torch.from_numpy(rows.view(np.int16).copy()).view(torch.bfloat16)
    A, s = bsg.quantize_fp8_rows(xt.cuda())
    torch.cuda.synchronize()
    A_ref, s_ref = oracle.quant_fp8_rows(rows)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(A.cpu().numpy(), A_ref)
    assert np.all(A_ref[1, :128] == 0)
    for gs in (np.float32(1e-30), np.float32(1e-3), np.float32(7.5e-41)):
        A4, sf = bsg.quantize_nvfp4_rows(xt.cuda(), torch.tensor([gs], dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        A4_ref, sf_ref = oracle.quant_nvfp4_rows(rows, gs)
        assert np.array_equal(sf.cpu().numpy(), sf_ref), f"gs {gs!r}"
        assert np.array_equal(A4.cpu().numpy(), A4_ref), f"gs {gs!r}"


def test_every_bf16_block_maximum():
    """Blocks whose maximum takes every positive bf16 value (the scale divisions amax / 448 and
    amax / 6 are computed without a division instruction): scales and codes bit-exact."""
    rng = np.random.default_rng(50)
    amax_bits = np.arange(0x0001, 0x7F80, dtype=np.uint16)
    # FP8: 128-element blocks, 128 blocks per row
    n = ((amax_bits.size + 127) // 128) * 128
    am = np.resize(amax_bits, n)
    blocks = (rng.uniform(-1, 1, (n, 128)).astype(np.float32)
              * (am.astype(np.uint32) << 16).view(np.float32)[:, None]).astype(np.float32)
    bits16 = (blocks.view(np.uint32) >> 16).astype(np.uint16)
    bits16[:, 0] = am
    rows = bits16.reshape(-1, 128 * 128)
    xt = torch.from_numpy(rows.view(np.int16).copy()).view(torch.bfloat16)
    A, s = bsg.quantize_fp8_rows(xt.cuda())
    torch.cuda.synchronize()
    A_ref, s_ref = oracle.quant_fp8_rows(rows)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(A.cpu().numpy(), A_ref)
    # NVFP4: 16-element blocks, 1024 blocks per row, two global scales
    n = ((amax_bits.size + 1023) // 1024) * 1024
    am = np.resize(amax_bits, n)
    blocks = (rng.uniform(-1, 1, (n, 16)).astype(np.float32)
              * (am.astype(np.uint32) << 16).view(np.float32)[:, None]).astype(np.float32)
    bits16 = (blocks.view(np.uint32) >> 16).astype(np.uint16)
    bits16[:, 0] = am
    rows = bits16.reshape(-1, 16 * 1024)
    xt = torch.from_numpy(rows.view(np.int16).copy()).view(torch.bfloat16)
    for gs in (np.float32(1.0 / 2688.0), np.float32(3.1e-7), np.float32(1.7e-30)):
        A4, sf = bsg.quantize_nvfp4_rows(xt.cuda(), torch.tensor([gs], dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        A4_ref, sf_ref = oracle.quant_nvfp4_rows(rows, gs)
        assert np.array_equal(sf.cpu().numpy(), sf_ref), f"gs {gs!r}"
        assert np.array_equal(A4.cpu().numpy(), A4_ref), f"gs {gs!r}"
