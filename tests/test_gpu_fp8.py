"""GPU parity of the FP8 grouped GEMM (through the C ABI) against the fp64 oracle.

Routing (which rows are written) is checked bit for bit with a sentinel-filled C; values within
max|gpu - ref| / (|ref| + rms(ref)) <= 8e-3.  Exact integer grids must match bit for bit.
"""
import numpy as np
import pytest
import torch

import nvfp4_grouped_gemm_indices_b200 as bsg
from nvfp4_grouped_gemm_indices_b200 import workloads as W

from gpu_util import (SENTINEL, DevWorkload, bits, compare, oracle_rows, routed_mask, sample_rows,
                      sentinel_out, to_dev)

pytestmark = pytest.mark.gpu

FP8_TACTICS = [0, 1, 2, 3, 4]  # 0: one SM per 128 x 256 tile; 1: an SM pair per 256 x 256 tile (cta_group::2);
# 2, 3: operand-swapped tiles (128 or 256 output columns x a chunk of at most 128 or 64 tokens);
# 4: one SM per 128 x 64 tile (small problems)


@pytest.fixture(params=FP8_TACTICS, ids=lambda t: f"tactic{t}")
def tactic(request):
    if request.param >= bsg.bsg_num_tactics(0):
        pytest.skip("tactic not built")
    bsg.bsg_set_tactic(0, request.param)
    yield request.param
    bsg.bsg_set_tactic(0, -1)


def full_check(w):
    d = DevWorkload(w)
    out = bits(d.run())
    torch.cuda.synchronize()
    bsg.bsg_get_device_status()
    ref = oracle_rows(w)
    return compare(out, ref, routed_mask(w))


def test_fp8_small_workload_full(tactic):
    """4 experts, M=512, N=256, K=512; run boundaries inside 128-row windows."""
    full_check(W.config(0))


@pytest.mark.parametrize("M,N,K,G,ctas", [(65, 128, 128, 2, 4), (777, 256, 512, 8, 84)])
def test_fp8_page_benchmark_shapes(M, N, K, G, ctas, tactic):
    """The two shapes of the FP8 page's benchmark table, balanced sorted runs."""
    counts = [M // G + (1 if i < M % G else 0) for i in range(G)]
    w = W.make_fp8(M, N, K, G, W.counts_to_indices(counts), seed=M)
    full_check(w)


def _routing(case, M, G, rng):
    if case == "sorted":
        return W.counts_to_indices(rng.multinomial(M, [1.0 / G] * G))
    if case == "len1_runs":
        return (np.arange(M) % G).astype(np.int32)
    if case == "empty_experts":
        counts = np.zeros(G, np.int64)
        counts[[1, G - 1]] = [M // 2, M - M // 2]
        return W.counts_to_indices(counts)
    if case == "span3windows":
        idx = np.full(M, -1, np.int32)
        idx[10:390] = 1
        idx[390:] = 0
        return idx
    if case == "skip_rows":
        idx = W.counts_to_indices(rng.multinomial(M, [1.0 / G] * G))
        idx[rng.random(M) < 0.2] = -1
        idx[rng.random(M) < 0.05] = G + 3
        return idx
    if case == "unsorted":
        return rng.integers(0, G, M).astype(np.int32)
    raise ValueError(case)


@pytest.mark.parametrize("case", ["sorted", "len1_runs", "empty_experts", "span3windows", "skip_rows", "unsorted"])
def test_fp8_routing_edge_cases(case, tactic):
    rng = np.random.default_rng(hash(case) % 1000)
    M, N, K, G = 400, 256, 256, 5
    w = W.make_fp8(M, N, K, G, _routing(case, M, G, rng), seed=7)
    full_check(w)


@pytest.mark.parametrize("M", [1, 127, 128, 129, 300])
def test_fp8_row_counts(M, tactic):
    G = 3 if M > 2 else 1
    rng = np.random.default_rng(M)
    idx = W.counts_to_indices(rng.multinomial(M, [1.0 / G] * G)) if G > 1 else np.zeros(M, np.int32)
    w = W.make_fp8(M, 256, 384, G, idx, seed=M)
    full_check(w)


def test_fp8_single_expert_null_indices(tactic):
    w = W.make_fp8(200, 256, 256, 1, None, seed=3)
    full_check(w)


@pytest.mark.parametrize("N", [64, 136, 264, 520])
def test_fp8_n_tails(N, tactic):
    rng = np.random.default_rng(N)
    idx = W.counts_to_indices(rng.multinomial(300, [0.5, 0.5]))
    w = W.make_fp8(300, N, 256, 2, idx, seed=N)
    full_check(w)


def test_fp8_many_experts_mostly_empty(tactic):
    """G = 64 with a Zipf routing of 512 rows: many experts with 0-3 rows."""
    rng = np.random.default_rng(11)
    idx = W.routing_zipf(512, 64, rng)
    w = W.make_fp8(512, 256, 512, 64, idx, seed=11)
    full_check(w)


def test_fp8_integer_grid_bit_exact(tactic):
    """Small integer codes and power-of-two scales: every sum is exact in fp32, so the GPU result
    must equal the oracle's bf16 bit for bit."""
    rng = np.random.default_rng(5)
    M, N, K, G = 300, 264, 512, 3
    pick = np.array([-1.0, 0.0, 0.0, 0.0, 0.0, 0.0, 1.0], np.float32)
    A = W.e4m3_encode(rng.choice(pick, (M, K)))
    B = W.e4m3_encode(rng.choice(pick, (G, N, K)))
    a_scale = np.exp2(rng.integers(-1, 2, (M, K // 128))).astype(np.float32)
    b_scale = np.exp2(rng.integers(-1, 2, (G, (N + 127) // 128, K // 128))).astype(np.float32)
    idx = W.counts_to_indices(rng.multinomial(M, [1 / 3] * 3))
    idx[::9] = -1
    w = W.Workload("grid", "fp8", M, N, K, G, A, B, idx, a_scale=a_scale, b_scale=b_scale)
    d = DevWorkload(w)
    out = bits(d.run())
    ref = oracle_rows(w)
    routed = routed_mask(w)
    assert np.array_equal(out[routed], ref[routed])
    assert np.all(out[~routed] == SENTINEL)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7])
def test_fp8_persistent_grid_sizes_bit_identical(ctas, tactic):
    """Each CTA walks many units through the same rings (stage counts that do not divide the
    number of K blocks): the result must not depend on the grid size."""
    rng = np.random.default_rng(21)
    idx = W.counts_to_indices(rng.multinomial(700, [0.2] * 5))
    w = W.make_fp8(700, 520, 640, 5, idx, seed=21)  # 5 K blocks, 4 stages; 3 N tiles
    d = DevWorkload(w)
    ref = bits(d.run())
    try:
        bsg.bsg_set_max_ctas(0, ctas)
        out = bits(d.run())
    finally:
        bsg.bsg_set_max_ctas(0, 0)
    assert np.array_equal(out, ref)
    compare(ref, oracle_rows(w), routed_mask(w))


def test_fp8_graph_replay_sees_new_indices(tactic):
    """m_indices is read on the device at every launch: a captured graph replayed after the routing
    (and the data) changed in place computes the new result."""
    rng = np.random.default_rng(8)
    M, N, K, G = 384, 256, 256, 4
    w1 = W.make_fp8(M, N, K, G, W.counts_to_indices(rng.multinomial(M, [0.25] * 4)), seed=1)
    idx2 = rng.integers(-1, G, M).astype(np.int32)
    w2 = W.make_fp8(M, N, K, G, idx2, seed=2)
    d = DevWorkload(w1)
    C = sentinel_out(M, N)
    s = torch.cuda.Stream()
    d.run(out=C, stream=s)  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        d.run(out=C, stream=s)
    C.view(torch.int16).fill_(SENTINEL)
    g.replay()
    torch.cuda.synchronize()
    compare(bits(C), oracle_rows(w1), routed_mask(w1))
    for name in ("A", "B", "a_scale", "b_scale", "m_indices"):
        getattr(d, name).copy_(to_dev(getattr(w2, name)))
    C.view(torch.int16).fill_(SENTINEL)
    g.replay()
    torch.cuda.synchronize()
    compare(bits(C), oracle_rows(w2), routed_mask(w2))


@pytest.mark.parametrize("cfg", [1, 4])
def test_fp8_full_size_sampled_rows(cfg, tactic):
    """The full-size FP8 workloads (MoE prefill G=8 M=8192 N=4096 K=7168; decode-like Zipf G=64
    M=512 N=4096 K=7168) in the benchmark's launch configuration, checked on every row near a run
    boundary plus random rows (all N columns); every other row is checked for NaN/sentinel."""
    w = W.config(cfg)
    d = DevWorkload(w)
    out = bits(d.run())
    bsg.bsg_get_device_status()
    rows = sample_rows(w, n_random=96, seed=cfg)
    compare(out[rows], oracle_rows(w, rows), routed_mask(w, rows))
    routed = routed_mask(w)
    assert np.all(out[~routed] == SENTINEL)
    assert not np.any((out[routed] & 0x7F80) == 0x7F80), "Inf/NaN in a routed row"


def test_fp8_bounded_wait_reports_timeout_and_context_survives():
    """Fault injection on the host side of the kernel: the scheduler withholds all work, every
    bounded wait expires (50 ms limit), the call reports BSG_ERR_DEVICE_TIMEOUT, nothing is written,
    and the next normal call on the same context is correct."""
    w = W.config(0)
    d = DevWorkload(w)
    prev = bsg.bsg_set_wait_timeout_ns(50_000_000)
    try:
        bsg.bsg_debug_set_fault(1)
        C = d.run()
        with pytest.raises(bsg.BsgError) as ei:
            bsg.bsg_get_device_status()
        assert ei.value.status == bsg.BSG_ERR_DEVICE_TIMEOUT
        assert np.all(bits(C) == SENTINEL)
    finally:
        bsg.bsg_debug_set_fault(0)
        bsg.bsg_set_wait_timeout_ns(prev)
    out = bits(d.run())
    bsg.bsg_get_device_status()
    compare(out, oracle_rows(w), routed_mask(w))


def test_fp8_autotune_under_expired_waits_records_nothing():
    """Autotune while every bounded wait expires (host-side fault injection, 50 ms limit): the
    launches return early and would look fastest, so the tuning must report BSG_ERR_DEVICE_TIMEOUT
    and record no tactic; the context stays usable."""
    w = W.config(0)
    d = DevWorkload(w)
    C = sentinel_out(w.M, w.N)
    bsg.bsg_autotune_clear()
    prev = bsg.bsg_set_wait_timeout_ns(50_000_000)
    try:
        bsg.bsg_debug_set_fault(1)
        with pytest.raises(bsg.BsgError) as ei:
            bsg.bsg_autotune_fp8(d.A, d.B, d.a_scale, d.b_scale, d.m_indices, C, w.M, w.N, w.K, w.G, reps=1)
        assert ei.value.status == bsg.BSG_ERR_DEVICE_TIMEOUT
    finally:
        bsg.bsg_debug_set_fault(0)
        bsg.bsg_set_wait_timeout_ns(prev)
    with pytest.raises(bsg.BsgError):
        bsg.bsg_get_device_status()                     # the word stayed set for the caller to see
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    forced_free = bsg.bsg_choose_tactic(0, w.M, w.N, w.K, w.G, sms)
    bsg.bsg_autotune_clear()
    assert forced_free == bsg.bsg_choose_tactic(0, w.M, w.N, w.K, w.G, sms)   # nothing was recorded
    out = bits(d.run())
    bsg.bsg_get_device_status()
    compare(out, oracle_rows(w), routed_mask(w))


def test_fp8_torch_wrapper():
    w = W.config(0)
    d = DevWorkload(w)
    C = bsg.fp8_grouped_gemm(d.A, d.B, d.a_scale, d.b_scale, d.m_indices)
    ref = oracle_rows(w)
    routed = routed_mask(w)
    out = bits(C)
    out[~routed] = SENTINEL  # the wrapper's fresh C is zero-filled
    compare(out, ref, routed)


def test_fp8_autotune_records_the_measured_winner_and_stays_correct():
    """Runtime autotune: every tactic runs on the caller's operands, the fastest is recorded for these
    sizes and picked by the chooser afterwards; C holds the correct result."""
    w = W.make_fp8(1024, 1024, 1024, 4, W.counts_to_indices([256, 300, 200, 268]), seed=44)
    d = DevWorkload(w)
    C = sentinel_out(w.M, w.N)
    bsg.bsg_autotune_clear()
    try:
        t = bsg.bsg_autotune_fp8(d.A, d.B, d.a_scale, d.b_scale, d.m_indices, C, w.M, w.N, w.K, w.G, reps=5)
        torch.cuda.synchronize()
        assert 0 <= t < bsg.bsg_num_tactics(0)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert bsg.bsg_choose_tactic(0, w.M, w.N, w.K, w.G, sms) == t
        compare(bits(C), oracle_rows(w), routed_mask(w))
    finally:
        bsg.bsg_autotune_clear()


def test_fp8_no_routed_rows_writes_nothing(tactic):
    """Every index out of range: the kernel hands out no unit and C stays untouched."""
    M, N, K, G = 300, 256, 256, 3
    idx = np.full(M, -1, np.int32)
    idx[::7] = G + 5
    w = W.make_fp8(M, N, K, G, idx, seed=9)
    out = bits(DevWorkload(w).run())
    bsg.bsg_get_device_status()
    assert np.all(out == SENTINEL)


def test_fp8_max_rows_and_max_experts():
    """The launch contract's extremes: M = 2^24 rows (two experts, a run boundary off the window
    grid) checked on sampled rows, and G = 4096 experts with one row each for a few of them."""
    M, N, K, G = 1 << 24, 64, 128, 2
    rng = np.random.default_rng(77)
    A = rng.integers(0, 0x7E, (M, K), dtype=np.uint8)          # finite E4M3 codes
    B = rng.integers(0, 0x7E, (G, N, K), dtype=np.uint8)
    a_scale = rng.uniform(0.5, 2.0, (M, 1)).astype(np.float32)
    b_scale = rng.uniform(0.5, 2.0, (G, 1, 1)).astype(np.float32)
    idx = np.zeros(M, np.int32)
    idx[(M // 2) + 37:] = 1
    w = W.Workload("fp8_max_m", "fp8", M, N, K, G, A, B, idx, a_scale=a_scale, b_scale=b_scale)
    d = DevWorkload(w)
    out = bits(d.run())
    bsg.bsg_get_device_status()
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(M // 2, M // 2 + 128), np.arange(M - 64, M),
                                     rng.integers(0, M, 256)]))
    compare(out[rows], oracle_rows(w, rows), routed_mask(w, rows))
    del d
    torch.cuda.empty_cache()
    G2, M2 = 4096, 600
    idx2 = np.full(M2, -1, np.int32)
    idx2[rng.choice(M2, 40, replace=False)] = rng.choice(G2, 40, replace=False).astype(np.int32)
    idx2 = np.sort(idx2)
    w2 = W.make_fp8(M2, 64, 128, G2, idx2, seed=78)
    compare(bits(DevWorkload(w2).run()), oracle_rows(w2), routed_mask(w2))
