"""Pins of the oracle's two GEMM definitions and of its window segmentation.

* exact integer grids: small integer codes and power-of-two scales make every sum exact and every
  result a bf16-representable dyadic number, compared bit for bit with an int64 library matmul;
* grouped == G dense GEMMs on the rows routed to each expert, bit for bit; unrouted rows untouched;
* exact rational brute force (``oracle.brute``) == oracle, bit for bit, including skip rows and the
  N-block boundary of the FP8 B scales;
* fp64 library matmul of operands decoded by an independent decoder == the oracle's unrounded sums
  to 1e-12 relative;
* the window-segment CTA counts printed on the FP8 page (tests/golden/fp8_window_program_ctas.txt).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from nvfp4_grouped_gemm_indices_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers


def lib_dec_e4m3(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


_E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], dtype=np.float64)


def lib_dec_e2m1_packed(packed):
    return _E2M1[W.unpack_e2m1(packed)]


def exact_bf16_bits(x):
    """bf16 bits of values that are exactly representable in bf16 (checked)."""
    x = np.asarray(x, dtype=np.float64)
    x32 = x.astype(np.float32)
    assert np.array_equal(x32.astype(np.float64), x)
    bits = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    back = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(back, x), "value not exactly representable in bf16"
    return bits


def random_fp8_case(M, N, K, G, seed, skip_frac=0.1):
    rng = np.random.default_rng(seed)
    A = W.e4m3_encode(rng.standard_normal((M, K)).astype(np.float32) * 4)
    B = W.e4m3_encode(rng.standard_normal((G, N, K)).astype(np.float32) * 4)
    NB = (N + 127) // 128
    a_scale = rng.uniform(0.001, 0.01, (M, K // 128)).astype(np.float32)
    b_scale = rng.uniform(0.001, 0.01, (G, NB, K // 128)).astype(np.float32)
    idx = rng.integers(0, G, M).astype(np.int32)
    idx[rng.random(M) < skip_frac] = -1
    idx[rng.random(M) < skip_frac / 2] = G  # also out of range on the high side
    return A, B, a_scale, b_scale, idx


def random_nvfp4_case(M, N, K, G, seed, skip_frac=0.1):
    rng = np.random.default_rng(seed)
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (G, N, K // 2), dtype=np.uint8)
    # non-negative finite E4M3 scale codes
    sfa = rng.integers(0x20, 0x48, (M, K // 16), dtype=np.uint8)
    sfb = rng.integers(0x20, 0x48, (G, N, K // 16), dtype=np.uint8)
    alpha = rng.uniform(0.5, 2.0, G).astype(np.float32)
    idx = rng.integers(0, G, M).astype(np.int32)
    idx[rng.random(M) < skip_frac] = -1
    return A, B, sfa, sfb, alpha, idx


# ----------------------------------------------------------------------------- exact integer grids


def int_grid_fp8(M, N, K, G, seed):
    rng = np.random.default_rng(seed)
    pick = np.array([-1.0, 0.0, 0.0, 0.0, 0.0, 0.0, 1.0], np.float32)
    vals = rng.choice(pick, size=(M, K))
    bvals = rng.choice(pick, size=(G, N, K))
    A = W.e4m3_encode(vals)
    B = W.e4m3_encode(bvals)
    NB = (N + 127) // 128
    a_scale = np.exp2(rng.integers(-1, 2, (M, K // 128))).astype(np.float32)
    b_scale = np.exp2(rng.integers(-1, 2, (G, NB, K // 128))).astype(np.float32)
    idx = rng.integers(0, G, M).astype(np.int32)
    idx[::7] = -1
    return A, B, a_scale, b_scale, idx, vals.astype(np.int64), bvals.astype(np.int64)


def test_fp8_integer_grid_exact():
    M, N, K, G = 33, 200, 256, 3
    A, B, sa, sb, idx, av, bv = int_grid_fp8(M, N, K, G, 1)
    out, f64 = oracle.fp8_grouped(A, B, sa, sb, idx, M, N, K, G, want_f64=True)
    KB = K // 128
    expect = np.zeros((M, N), np.float64)
    for m in range(M):
        g = idx[m]
        if g < 0 or g >= G:
            continue
        for kb in range(KB):
            sl = slice(kb * 128, kb * 128 + 128)
            part = bv[g][:, sl] @ av[m, sl]          # int64 library matmul, exact
            colscale = sb[g][np.arange(N) // 128, kb].astype(np.float64)
            expect[m] += float(sa[m, kb]) * colscale * part
    routed = (idx >= 0) & (idx < G)
    assert np.array_equal(f64[routed], expect[routed])
    assert np.array_equal(out[routed], exact_bf16_bits(expect[routed]))
    assert np.all(out[~routed] == 0xFFFF)


def test_nvfp4_integer_grid_exact():
    M, N, K, G = 21, 40, 128, 2
    rng = np.random.default_rng(2)
    # E2M1 codes of 0, +-1, +-2 only (mostly 0); scales 2^-1..2^1 (E4M3 codes 0x30, 0x38, 0x40);
    # alpha 2^-2 and 2^-1, so every result is a dyadic number with at most 8 significant bits
    choices = np.array([0, 0, 0, 0, 0, 0, 2, 4, 10, 12], np.uint8)  # 0, 1, 2, -1, -2
    av = rng.choice(choices, (M, K))
    bv = rng.choice(choices, (G, N, K))
    A = W.pack_e2m1(av)
    B = W.pack_e2m1(bv)
    sfa = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (M, K // 16))
    sfb = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (G, N, K // 16))
    alpha = np.array([0.25, 0.5], np.float32)
    idx = rng.integers(-1, G, M).astype(np.int32)
    out, f64 = oracle.nvfp4(A, B, sfa, sfb, alpha, idx, M, N, K, G, want_f64=True)
    ival = {0: 0, 2: 1, 4: 2, 10: -1, 12: -2}
    ai = np.vectorize(ival.get)(av).astype(np.int64)
    bi = np.vectorize(ival.get)(bv).astype(np.int64)
    sval = {0x30: 0.5, 0x38: 1.0, 0x40: 2.0}
    sa = np.vectorize(sval.get)(sfa)
    sb = np.vectorize(sval.get)(sfb)
    expect = np.zeros((M, N))
    for m in range(M):
        g = idx[m]
        if g < 0:
            continue
        for j in range(K // 16):
            sl = slice(j * 16, j * 16 + 16)
            expect[m] += sa[m, j] * sb[g][:, j] * (bi[g][:, sl] @ ai[m, sl])
        expect[m] *= float(alpha[g])
    routed = idx >= 0
    assert np.array_equal(f64[routed], expect[routed])
    assert np.array_equal(out[routed], exact_bf16_bits(expect[routed]))
    assert np.all(out[~routed] == 0xFFFF)


# ----------------------------------------------------------------------------- grouped == dense


def test_fp8_grouped_equals_dense_per_expert():
    M, N, K, G = 300, 136, 384, 3
    A, B, sa, sb, idx = random_fp8_case(M, N, K, G, 3)
    grouped, _ = oracle.fp8_grouped(A, B, sa, sb, idx, M, N, K, G)
    for g in range(G):
        rows = np.nonzero(idx == g)[0]
        dense, _ = oracle.fp8_grouped(A[rows], B[g:g + 1], sa[rows], sb[g:g + 1], None, len(rows), N, K, 1)
        assert np.array_equal(grouped[rows], dense)
    unrouted = (idx < 0) | (idx >= G)
    assert unrouted.any() and np.all(grouped[unrouted] == 0xFFFF)


def test_nvfp4_grouped_equals_dense_per_expert():
    M, N, K, G = 200, 72, 256, 4
    A, B, sfa, sfb, alpha, idx = random_nvfp4_case(M, N, K, G, 4)
    grouped, _ = oracle.nvfp4(A, B, sfa, sfb, alpha, idx, M, N, K, G)
    for g in range(G):
        rows = np.nonzero(idx == g)[0]
        dense, _ = oracle.nvfp4(A[rows], B[g:g + 1], sfa[rows], sfb[g:g + 1], alpha[g:g + 1], None,
                                len(rows), N, K, 1)
        assert np.array_equal(grouped[rows], dense)
    assert np.all(grouped[idx < 0] == 0xFFFF)


def test_row_subset_matches_full():
    M, N, K, G = 64, 40, 256, 2
    A, B, sa, sb, idx = random_fp8_case(M, N, K, G, 5)
    full, _ = oracle.fp8_grouped(A, B, sa, sb, idx, M, N, K, G)
    rows = np.array([63, 0, 17, 17, 5])
    sub, _ = oracle.fp8_grouped(A, B, sa, sb, idx, M, N, K, G, rows=rows)
    assert np.array_equal(sub, full[rows])


# ----------------------------------------------------------------------------- brute force


@pytest.mark.parametrize("seed", [0, 1])
def test_fp8_matches_exact_brute_force(seed):
    M, N, K, G = 5, 132, 256, 3   # N crosses the 128-column block of b_scale
    A, B, sa, sb, idx = random_fp8_case(M, N, K, G, 10 + seed, skip_frac=0.2)
    idx[0] = -1
    ours, _ = oracle.fp8_grouped(A, B, sa, sb, idx, M, N, K, G)
    ref = brute.fp8_grouped(A, B, sa, sb, idx, M, N, K, G)
    for (m, n), bits in ref.items():
        assert int(ours[m, n]) == bits, (m, n)
    for m in range(M):
        if not (0 <= idx[m] < G):
            assert np.all(ours[m] == 0xFFFF)


@pytest.mark.parametrize("seed", [0, 1])
def test_nvfp4_matches_exact_brute_force(seed):
    M, N, K, G = 6, 16, 64, 3
    A, B, sfa, sfb, alpha, idx = random_nvfp4_case(M, N, K, G, 20 + seed, skip_frac=0.2)
    idx[1] = -1
    ours, _ = oracle.nvfp4(A, B, sfa, sfb, alpha, idx, M, N, K, G)
    ref = brute.nvfp4(A, B, sfa, sfb, alpha, idx, M, N, K, G)
    for (m, n), bits in ref.items():
        assert int(ours[m, n]) == bits, (m, n)
    assert np.all(ours[1] == 0xFFFF)


# ----------------------------------------------------------------------------- library fp64 matmul


def test_fp8_unrounded_matches_library_matmul():
    w = W.make_fp8(160, 256, 512, 3, W.counts_to_indices([50, 0, 110]), seed=31)
    M, N, K, G = w.M, w.N, w.K, w.G
    _, f64 = oracle.fp8_grouped(w.A, w.B, w.a_scale, w.b_scale, w.m_indices, M, N, K, G, want_f64=True)
    Ad = lib_dec_e4m3(w.A)
    expect = np.zeros((M, N))
    for kb in range(K // 128):
        sl = slice(kb * 128, kb * 128 + 128)
        for g in range(G):
            rows = np.nonzero(w.m_indices == g)[0]
            if rows.size == 0:
                continue
            Bd = lib_dec_e4m3(w.B[g][:, sl])
            part = Ad[rows][:, sl] @ Bd.T
            colscale = w.b_scale[g][np.arange(N) // 128, kb].astype(np.float64)
            expect[rows] += w.a_scale[rows, kb].astype(np.float64)[:, None] * colscale[None, :] * part
    np.testing.assert_allclose(f64, expect, rtol=1e-12, atol=1e-300)


def test_nvfp4_unrounded_matches_library_matmul():
    w = W.make_nvfp4(96, 64, 256, 2, W.counts_to_indices([40, 56]), seed=32)
    M, N, K, G = w.M, w.N, w.K, w.G
    _, f64 = oracle.nvfp4(w.A, w.B, w.sfa, w.sfb, w.alpha, w.m_indices, M, N, K, G, want_f64=True)
    Ad = lib_dec_e2m1_packed(w.A)
    sa = lib_dec_e4m3(w.sfa)
    expect = np.zeros((M, N))
    for g in range(G):
        rows = np.nonzero(w.m_indices == g)[0]
        Bd = lib_dec_e2m1_packed(w.B[g])
        sb = lib_dec_e4m3(w.sfb[g])
        for j in range(K // 16):
            sl = slice(j * 16, j * 16 + 16)
            expect[rows] += sa[rows, j][:, None] * sb[:, j][None, :] * (Ad[rows][:, sl] @ Bd[:, sl].T)
        expect[rows] *= float(w.alpha[g])
    np.testing.assert_allclose(f64, expect, rtol=1e-12, atol=1e-300)


# ----------------------------------------------------------------------------- window plan


def _golden_ctas():
    rows = []
    with open(os.path.join(GOLDEN, "fp8_window_program_ctas.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, M, N, K, G, ctas = line.split()
                rows.append((name, int(M), int(N), int(K), int(G), int(ctas)))
    return rows


@pytest.mark.parametrize("case", _golden_ctas(), ids=lambda c: c[0])
def test_window_program_cta_count_matches_printed_table(case):
    """The printed CTA counts follow from ceil(M/128) x (largest number of per-expert segments in a
    window) x ceil(N/64), for balanced sorted runs that start inside windows."""
    name, M, N, K, G, ctas = case
    counts = [M // G + (1 if i < M % G else 0) for i in range(G)]
    idx = W.counts_to_indices(counts)
    assert oracle.window_grid_ctas(idx, M, N, G) == ctas
    # the alternative reading (one CTA per segment, summed over windows) does not reproduce it
    segs = oracle.window_plan(idx, M, G)
    assert len(segs) * ((N + 63) // 64) != ctas or M <= 128


def test_window_plan_segments():
    idx = np.array([0] * 100 + [1] * 40 + [-1] * 3 + [1] * 10 + [2] * 150 + [5] * 3, np.int32)
    M = idx.size
    segs = oracle.window_plan(idx, M, 3)
    assert segs == [(0, 0, 100, 0), (0, 100, 128, 1), (1, 128, 140, 1), (1, 143, 153, 1),
                    (1, 153, 256, 2), (2, 256, 303, 2)]
    # every routed row is covered exactly once, every segment inside one window, one expert
    covered = np.zeros(M, int)
    for (w, lo, hi, g) in segs:
        assert w * 128 <= lo < hi <= (w + 1) * 128
        assert np.all(idx[lo:hi] == g)
        covered[lo:hi] += 1
    assert np.array_equal(covered, ((idx >= 0) & (idx < 3)).astype(int))
