"""GPU parity of the MoE expand permutation (through the C ABI) against the oracle's stable counting
sort: every output (src_rows, m_indices, dst_rows, expert_offsets) is integer data and must match
bit for bit; and the whole expand chain (permute -> quantise with the gather -> grouped GEMM)
against the oracle's chain."""
import numpy as np
import pytest
import torch

import nvfp4_grouped_gemm_indices_b200 as bsg
from nvfp4_grouped_gemm_indices_b200 import workloads as W
import oracle
from gpu_util import SENTINEL, bits, compare

pytestmark = pytest.mark.gpu


def make_ids(T, top_k, G, seed, invalid=0.0, zipf=False):
    rng = np.random.default_rng(seed)
    if zipf:
        ranks = np.arange(1, G + 1, dtype=np.float64) ** -1.2
        p = ranks / ranks.sum()
        ids = rng.choice(G, size=(T, top_k), p=p[rng.permutation(G)]).astype(np.int32)
    else:
        ids = rng.integers(0, G, (T, top_k)).astype(np.int32)
    if invalid > 0:
        bad = rng.random((T, top_k)) < invalid
        ids[bad] = rng.choice(np.array([-1, -9, G, G + 11], np.int32), int(bad.sum()))
    return ids


def run_permute(ids, G, ws=None, garbage=True):
    T, top_k = ids.shape
    n = T * top_k
    nbytes = bsg.bsg_moe_permute_workspace_size(T, top_k, G)
    if ws is None:
        ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device="cuda")
    if garbage:
        ws.fill_(0xA5)                               # the scratch needs no initialisation
    e = torch.from_numpy(ids).cuda()
    src = torch.full((n,), 0x5EED, dtype=torch.int32, device="cuda")
    mi = torch.full((n,), 0x5EED, dtype=torch.int32, device="cuda")
    dst = torch.full((T, top_k), 0x5EED, dtype=torch.int32, device="cuda")
    off = torch.full((G + 1,), 0x5EED, dtype=torch.int32, device="cuda")
    bsg.bsg_moe_permute(e, T, top_k, G, src, mi, dst, off, ws, ws.numel())
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (src, mi, dst, off)]


def check(ids, G, got):
    ref = oracle.moe_permute(ids, G)
    for name, a, b in zip(("src_rows", "m_indices", "dst_rows", "expert_offsets"), got, ref):
        assert np.array_equal(a, b), f"{name} differs at {np.nonzero(a != b)[0][:8]}"


@pytest.mark.parametrize("T,top_k,G,invalid,zipf", [
    (1, 1, 1, 0.0, False), (37, 3, 5, 0.2, False), (8192, 8, 8, 0.0, False), (4096, 6, 256, 0.0, True),
    (1000, 2, 4096, 0.05, False), (50, 4, 3, 1.0, False), (65536, 8, 64, 0.01, True), (257, 1, 2, 0.0, False),
    # the single-CTA path's limits (4096 entries, 1024 experts) and the first sizes past them
    (512, 8, 1024, 0.01, True), (9, 7, 1024, 0.0, False), (4097, 1, 8, 0.0, True), (64, 2, 1025, 0.1, False),
    (2048, 32, 1024, 0.01, True), (1 << 18, 1, 5, 0.0, True),
])
def test_permute_bit_exact(T, top_k, G, invalid, zipf):
    ids = make_ids(T, top_k, G, seed=T * 7 + G, invalid=invalid, zipf=zipf)
    check(ids, G, run_permute(ids, G))


def test_permute_largest_size():
    """T * top_k = 2^24 entries over 4096 experts: 512 tiles of 32768 entries (8 MiB of counters)."""
    T, top_k, G = 1 << 21, 8, 4096
    ids = make_ids(T, top_k, G, seed=5, invalid=0.001, zipf=True)
    check(ids, G, run_permute(ids, G))


def test_permute_calls_in_a_row_share_the_workspace():
    G = 32                                   # 80000 entries: the three-launch path, with scratch
    ws = torch.empty(bsg.bsg_moe_permute_workspace_size(20000, 4, G), dtype=torch.uint8, device="cuda")
    assert ws.numel() > 0
    for seed in range(3):
        ids = make_ids(20000, 4, G, seed=seed, invalid=0.1)
        check(ids, G, run_permute(ids, G, ws=ws, garbage=False))


@pytest.mark.parametrize("T", [500, 20000])
def test_permute_graph_replay_sees_new_routing(T):
    """No allocation and no host read in the call: it captures into a CUDA graph, and a replay after
    the routing changed in place gives the new permutation (single-CTA and three-launch sizes)."""
    top_k, G = 4, 16
    n = T * top_k
    ids0 = make_ids(T, top_k, G, seed=1)
    e = torch.from_numpy(ids0).cuda()
    ws = torch.empty(max(16, bsg.bsg_moe_permute_workspace_size(T, top_k, G)), dtype=torch.uint8, device="cuda")
    outs = [torch.empty(n, dtype=torch.int32, device="cuda"), torch.empty(n, dtype=torch.int32, device="cuda"),
            torch.empty((T, top_k), dtype=torch.int32, device="cuda"),
            torch.empty(G + 1, dtype=torch.int32, device="cuda")]
    s = torch.cuda.Stream()
    bsg.bsg_moe_permute(e, T, top_k, G, *outs, ws, ws.numel(), s)   # first call outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        bsg.bsg_moe_permute(e, T, top_k, G, *outs, ws, ws.numel(), s)
    for seed in (2, 3):
        ids = make_ids(T, top_k, G, seed=seed, invalid=0.05)
        e.copy_(torch.from_numpy(ids))
        g.replay()
        torch.cuda.synchronize()
        check(ids, G, [t.cpu().numpy() for t in outs])


def test_permute_torch_wrapper():
    ids = make_ids(500, 2, 12, seed=9, invalid=0.1)
    got = bsg.moe_permute(torch.from_numpy(ids).cuda(), 12)
    check(ids, 12, [t.cpu().numpy() for t in got])


@pytest.mark.parametrize("kind", ["fp8", "nvfp4"])
def test_expand_chain_matches_the_oracle_chain(kind):
    """Routing -> expand permutation -> quantise the gathered activations -> grouped GEMM, all on the
    GPU, against the oracle's permutation feeding the oracle's quantiser feeding the oracle's GEMM.
    The permutation and the codes are integers (bit-exact); C is within the GEMM tolerance, with the
    rows of dropped entries (m_indices -1) left untouched."""
    rng = np.random.default_rng(60)
    T, top_k, G, N, K = 700, 3, 6, 256, 512
    ids = make_ids(T, top_k, G, seed=61, invalid=0.05)
    n = T * top_k
    x = (rng.standard_normal((T, K)).astype(np.float32) * 3).astype(np.float32)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    xb = xt.view(torch.int16).numpy().view(np.uint16)
    src, mi, dst, off = bsg.moe_permute(torch.from_numpy(ids).cuda(), G)
    src_r, mi_r, dst_r, off_r = oracle.moe_permute(ids, G)
    assert np.array_equal(src.cpu().numpy(), src_r) and np.array_equal(mi.cpu().numpy(), mi_r)
    C = torch.full((n, N), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    routed = (mi_r >= 0)
    if kind == "fp8":
        w = W.make_fp8(n, N, K, G, mi_r, seed=62)                   # the experts' B and b_scale
        A = torch.full((n, K), 0, dtype=torch.uint8, device="cuda")
        s = torch.full((n, K // 128), 0, dtype=torch.float32, device="cuda")
        bsg.bsg_quantize_fp8_rows(xt.cuda(), src, A, s, T, n, K)
        bsg.fp8_grouped_gemm(A, torch.from_numpy(w.B).cuda(), s, torch.from_numpy(w.b_scale).cuda(), mi, out=C)
        torch.cuda.synchronize()
        A_r, s_r = oracle.quant_fp8_rows(xb, M=n, src_rows=src_r, A=np.zeros((n, K), np.uint8),
                                         scale=np.zeros((n, K // 128), np.float32))
        assert np.array_equal(A.cpu().numpy(), A_r)
        ref, _ = oracle.fp8_grouped(A_r, w.B, s_r, w.b_scale, mi_r, n, N, K, G)
    else:
        w = W.make_nvfp4(n, N, K, G, mi_r, seed=63)
        gs = W.nvfp4_global_scale(x)
        A = torch.full((n, K // 2), 0, dtype=torch.uint8, device="cuda")
        sf = torch.full((n, K // 16), 0, dtype=torch.uint8, device="cuda")
        bsg.bsg_quantize_nvfp4_rows(xt.cuda(), src, torch.tensor([gs], device="cuda"), A, sf, T, n, K)
        bsg.nvfp4_gemm(A, torch.from_numpy(w.B).cuda(), sf, torch.from_numpy(w.sfb).cuda(),
                       torch.from_numpy(w.alpha).cuda(), mi, out=C)
        torch.cuda.synchronize()
        A_r, sf_r = oracle.quant_nvfp4_rows(xb, gs, M=n, src_rows=src_r, A=np.zeros((n, K // 2), np.uint8),
                                            sf=np.zeros((n, K // 16), np.uint8))
        assert np.array_equal(A.cpu().numpy(), A_r) and np.array_equal(sf.cpu().numpy(), sf_r)
        ref, _ = oracle.nvfp4(A_r, w.B, sf_r, w.sfb, w.alpha, mi_r, n, N, K, G)
    compare(bits(C), ref, routed)
