"""GPU parity of the NVFP4 (grouped) GEMM (through the C ABI) against the fp64 oracle.

Routing is checked bit for bit with a sentinel-filled C; values within
max|gpu - ref| / (|ref| + rms(ref)) <= 8e-3; exact integer grids bit for bit.
"""
import numpy as np
import pytest
import torch

import nvfp4_grouped_gemm_indices_b200 as bsg
from nvfp4_grouped_gemm_indices_b200 import workloads as W

from gpu_util import (SENTINEL, DevWorkload, bits, compare, oracle_rows, routed_mask, sample_rows,
                      sentinel_out, to_dev)

pytestmark = pytest.mark.gpu

NVFP4_TACTICS = [0, 1]  # 0: one SM per 128 x 256 tile; 1: an SM pair per 256 x 256 tile (cta_group::2)


@pytest.fixture(params=NVFP4_TACTICS, ids=lambda t: f"tactic{t}", autouse=True)
def tactic(request):
    if request.param >= bsg.bsg_num_tactics(1):
        pytest.skip("tactic not built")
    bsg.bsg_set_tactic(1, request.param)
    yield request.param
    bsg.bsg_set_tactic(1, -1)


def full_check(w):
    d = DevWorkload(w)
    out = bits(d.run())
    torch.cuda.synchronize()
    bsg.bsg_get_device_status()
    return compare(out, oracle_rows(w), routed_mask(w))


def test_nvfp4_small_dense():
    w = W.make_nvfp4(256, 256, 512, 1, None, seed=1)
    full_check(w)


def test_nvfp4_small_grouped():
    rng = np.random.default_rng(2)
    idx = W.routing_multinomial_unaligned(512, 4, rng)
    w = W.make_nvfp4(512, 512, 1024, 4, idx, seed=2)
    full_check(w)


@pytest.mark.parametrize("case", ["len1_runs", "empty_experts", "skip_rows", "unsorted"])
def test_nvfp4_routing_edge_cases(case):
    rng = np.random.default_rng(len(case))
    M, G = 300, 4
    if case == "len1_runs":
        idx = (np.arange(M) % G).astype(np.int32)
    elif case == "empty_experts":
        idx = W.counts_to_indices([0, 150, 0, 150])
    elif case == "skip_rows":
        idx = W.counts_to_indices(rng.multinomial(M, [0.25] * 4))
        idx[rng.random(M) < 0.25] = -1
    else:
        idx = rng.integers(0, G, M).astype(np.int32)
    w = W.make_nvfp4(M, 256, 512, G, idx, seed=5)
    full_check(w)


@pytest.mark.parametrize("M,N,K", [(1, 64, 256), (129, 136, 256), (200, 520, 768)])
def test_nvfp4_shapes_and_tails(M, N, K):
    w = W.make_nvfp4(M, N, K, 1, np.zeros(M, np.int32), seed=M + N)
    full_check(w)


def test_nvfp4_integer_grid_bit_exact():
    rng = np.random.default_rng(9)
    M, N, K, G = 200, 264, 512, 2
    choices = np.array([0, 0, 0, 0, 0, 0, 2, 4, 10, 12], np.uint8)  # 0, +-1, +-2
    A = W.pack_e2m1(rng.choice(choices, (M, K)))
    B = W.pack_e2m1(rng.choice(choices, (G, N, K)))
    sfa = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (M, K // 16))
    sfb = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (G, N, K // 16))
    alpha = np.array([0.25, 0.5], np.float32)
    idx = rng.integers(-1, G, M).astype(np.int32)
    w = W.Workload("grid", "nvfp4", M, N, K, G, A, B, idx, sfa=sfa, sfb=sfb, alpha=alpha)
    d = DevWorkload(w)
    out = bits(d.run())
    ref = oracle_rows(w)
    routed = routed_mask(w)
    assert np.array_equal(out[routed], ref[routed])
    assert np.all(out[~routed] == SENTINEL)


def test_nvfp4_one_scale_per_block_is_applied():
    """Only one 16-element block of one row/column carries a non-unit scale: catches a scale-factor
    layout error (a scale applied to the wrong block, row or column)."""
    M, N, K, G = 128, 256, 512, 1
    rng = np.random.default_rng(4)
    A = W.pack_e2m1(rng.choice(np.array([2, 10], np.uint8), (M, K)))    # +-1
    B = W.pack_e2m1(rng.choice(np.array([2, 10], np.uint8), (G, N, K)))
    for (r, j, code) in [(5, 3, 0x40), (77, 17, 0x30), (127, 31, 0x48)]:
        sfa = np.full((M, K // 16), 0x38, np.uint8)
        sfb = np.full((G, N, K // 16), 0x38, np.uint8)
        sfa[r, j] = code
        sfb[0, (r * 3) % N, (j + 5) % (K // 16)] = code
        w = W.Workload("sf", "nvfp4", M, N, K, G, A, B, np.zeros(M, np.int32), sfa=sfa, sfb=sfb,
                       alpha=np.ones(1, np.float32))
        d = DevWorkload(w)
        out = bits(d.run())
        assert np.array_equal(out, oracle_rows(w))


@pytest.mark.parametrize("ctas", [1, 3, 7])
def test_nvfp4_persistent_grid_sizes_bit_identical(ctas):
    rng = np.random.default_rng(31)
    idx = W.counts_to_indices(rng.multinomial(600, [0.25] * 4))
    w = W.make_nvfp4(600, 520, 1280, 4, idx, seed=31)  # 5 K stages, 4-stage ring
    d = DevWorkload(w)
    ref = bits(d.run())
    try:
        bsg.bsg_set_max_ctas(1, ctas)
        out = bits(d.run())
    finally:
        bsg.bsg_set_max_ctas(1, 0)
    assert np.array_equal(out, ref)
    compare(ref, oracle_rows(w), routed_mask(w))


def test_nvfp4_graph_replay_sees_new_indices():
    rng = np.random.default_rng(12)
    M, N, K, G = 256, 256, 512, 3
    w1 = W.make_nvfp4(M, N, K, G, W.counts_to_indices(rng.multinomial(M, [1 / 3] * 3)), seed=1)
    w2 = W.make_nvfp4(M, N, K, G, rng.integers(-1, G, M).astype(np.int32), seed=2)
    d = DevWorkload(w1)
    C = sentinel_out(M, N)
    s = torch.cuda.Stream()
    d.run(out=C, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        d.run(out=C, stream=s)
    C.view(torch.int16).fill_(SENTINEL)
    g.replay()
    torch.cuda.synchronize()
    compare(bits(C), oracle_rows(w1), routed_mask(w1))
    for name in ("A", "B", "sfa", "sfb", "alpha", "m_indices"):
        getattr(d, name).copy_(to_dev(getattr(w2, name)))
    C.view(torch.int16).fill_(SENTINEL)
    g.replay()
    torch.cuda.synchronize()
    compare(bits(C), oracle_rows(w2), routed_mask(w2))


@pytest.mark.parametrize("cfg", [2, 3])
def test_nvfp4_full_size_sampled_rows(cfg):
    """Full-size NVFP4 workloads (dense M=2048 N=36864 K=4608; grouped G=8 x 8192 rows, N=K=8192)
    checked on sampled rows (run boundaries + random), every other row for NaN/sentinel."""
    w = W.config(cfg)
    d = DevWorkload(w)
    out = bits(d.run())
    bsg.bsg_get_device_status()
    rows = sample_rows(w, n_random=24 if cfg == 3 else 48, seed=cfg)
    compare(out[rows], oracle_rows(w, rows), routed_mask(w, rows))
    routed = routed_mask(w)
    assert np.all(out[~routed] == SENTINEL)
    assert not np.any((out[routed] & 0x7F80) == 0x7F80), "Inf/NaN in a routed row"


def test_nvfp4_bounded_wait_reports_timeout_and_context_survives():
    w = W.make_nvfp4(256, 256, 512, 1, None, seed=1)
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
    full_check(w)


def test_nvfp4_autotune_records_the_measured_winner_and_stays_correct():
    rng = np.random.default_rng(45)
    w = W.make_nvfp4(512, 1024, 1024, 2, W.counts_to_indices(rng.multinomial(512, [0.5, 0.5])), seed=45)
    d = DevWorkload(w)
    C = sentinel_out(w.M, w.N)
    bsg.bsg_autotune_clear()
    try:
        bsg.bsg_set_tactic(1, -1)
        t = bsg.bsg_autotune_nvfp4(d.A, d.B, d.sfa, d.sfb, d.alpha, d.m_indices, C, w.M, w.N, w.K, w.G, reps=5)
        torch.cuda.synchronize()
        assert 0 <= t < bsg.bsg_num_tactics(1)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert bsg.bsg_choose_tactic(1, w.M, w.N, w.K, w.G, sms) == t
        compare(bits(C), oracle_rows(w), routed_mask(w))
    finally:
        bsg.bsg_autotune_clear()
