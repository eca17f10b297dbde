"""Seeded synthetic inputs for the block-scaled grouped GEMM.

This module only draws random numbers and quantises them into the operand formats the library
consumes; it performs none of the GEMM arithmetic.  Both the CUDA path (through the tests and the
benchmark) and the CPU oracle take their inputs from here.

Formats (bit layouts are those of the OCP 8-bit / 4-bit floating-point formats):

* E4M3 ("FN" flavour, largest finite 448, saturating quantiser as in the page "ROCm 아키텍처별
  최적화: 런타임 디스패치로 성능 극대화", section 1, which clamps to +-448 before converting);
* E2M1 (values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives), two codes per byte, the lower-K
  element in the low nibble;
* UE4M3 block scales for NVFP4 (E4M3 codes of non-negative values).

Quantisation recipes (the five workloads of the benchmark):

* FP8: per 1x128 K block of A and per 128x128 block of B[g]: ``scale = amax / 448`` (fp32),
  ``code = e4m3_rne_satfinite(x / scale)`` with the quotient one correctly rounded fp32 division;
  an all-zero block gets scale 0 and zero codes.
* NVFP4: ``gs = amax(tensor) / (448 * 6)``; per 16 K elements ``s = ue4m3_rne((amax16 / 6) / gs)``;
  ``code = e2m1_rne_satfinite(x / (s * gs))``; ``alpha[g] = gs_A * gs_B[g]`` (B's global scale is
  taken per expert, each B[g] being its own weight tensor).

Seeds: ``SeedSequence(seed)`` is spawned into three children for A, B and the routing, in that
order; A and B are drawn in 1024-row chunks (B: per expert and 128-row block), each chunk from its own
spawned ``PCG64`` stream, so the result does not depend on how many threads generate it.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0
E2M1_MAX = 6.0

# ----------------------------------------------------------------------------- element encoders


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 code, round to nearest even, saturating at +-448 (NaN stays NaN)."""
    x = np.asarray(x, dtype=np.float32)
    clipped = np.clip(x, -E4M3_MAX, E4M3_MAX)
    t = torch.from_numpy(np.ascontiguousarray(clipped)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 code -> fp32 through the library's float8 type (used for scale reconstruction only)."""
    c = torch.from_numpy(np.ascontiguousarray(np.asarray(codes, dtype=np.uint8)))
    return c.view(torch.float8_e4m3fn).to(torch.float32).numpy()


# E2M1 magnitudes in code order 0..7, and the decision points of round-to-nearest-even between
# neighbours (a tie goes to the neighbour with the even code).
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> E2M1 4-bit code (uint8 holding 0..15), RNE, saturating at +-6."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x)
    # midpoints between consecutive magnitudes; ties resolve toward the even code
    code = np.zeros(a.shape, dtype=np.uint8)
    code = np.where(a > 0.25, 1, code)      # 0.25 ties to 0 (code 0 even)
    code = np.where(a >= 0.75, 2, code)     # 0.75 ties to 1.0 (code 2 even)
    code = np.where(a > 1.25, 3, code)      # 1.25 ties to 1.0 (code 2)
    code = np.where(a >= 1.75, 4, code)     # 1.75 ties to 2.0 (code 4)
    code = np.where(a > 2.5, 5, code)       # 2.5 ties to 2.0 (code 4)
    code = np.where(a >= 3.5, 6, code)      # 3.5 ties to 4.0 (code 6)
    code = np.where(a > 5.0, 7, code)       # 5.0 ties to 4.0 (code 6)
    code = code.astype(np.uint8)
    sign = (np.signbit(x)).astype(np.uint8) << 3
    return (code | sign).astype(np.uint8)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """[..., K] nibble codes -> [..., K/2] bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# ----------------------------------------------------------------------------- quantisers


def quant_fp8_rows(x: np.ndarray):
    """Quantise [R, K] fp32 per 1x128 block.  Returns (codes uint8 [R,K], scale f32 [R,K/128])."""
    R, K = x.shape
    xb = x.reshape(R, K // 128, 128)
    amax = np.abs(xb).max(axis=-1).astype(np.float32)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (xb / safe[..., None]).astype(np.float32)          # one correctly rounded fp32 division
    codes = np.where((scale > 0)[..., None], e4m3_encode(q), np.uint8(0))
    return codes.astype(np.uint8).reshape(R, K), scale


def quant_fp8_blocks(w: np.ndarray):
    """Quantise [N, K] fp32 per 128x128 block (N tail block may be short).  Returns (codes [N,K],
    scale f32 [ceil(N/128), K/128])."""
    N, K = w.shape
    NB = (N + 127) // 128
    codes = np.empty((N, K), dtype=np.uint8)
    scale = np.empty((NB, K // 128), dtype=np.float32)
    for nb in range(NB):
        blk = w[nb * 128:(nb + 1) * 128].reshape(-1, K // 128, 128)
        amax = np.abs(blk).max(axis=(0, 2)).astype(np.float32)
        s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
        safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
        q = (blk / safe[None, :, None]).astype(np.float32)
        c = np.where((s > 0)[None, :, None], e4m3_encode(q), np.uint8(0)).astype(np.uint8)
        codes[nb * 128:(nb + 1) * 128] = c.reshape(-1, K)
        scale[nb] = s
    return codes, scale


def nvfp4_global_scale(x: np.ndarray) -> np.float32:
    amax = np.float32(np.abs(x).max()) if x.size else np.float32(0.0)
    return np.float32(amax / np.float32(E4M3_MAX * E2M1_MAX))


def quant_nvfp4(x: np.ndarray, gs: np.float32, chunk_rows: int = 4096):
    """Quantise [R, K] fp32 to NVFP4 with global scale ``gs``.  Returns (packed uint8 [R, K/2],
    sf uint8 [R, K/16] (UE4M3 codes))."""
    R, K = x.shape
    packed = np.empty((R, K // 2), dtype=np.uint8)
    sf = np.empty((R, K // 16), dtype=np.uint8)
    gs = np.float32(gs)
    for r0 in range(0, R, chunk_rows):
        xb = x[r0:r0 + chunk_rows].reshape(-1, K // 16, 16)
        amax16 = np.abs(xb).max(axis=-1).astype(np.float32)
        if gs > 0:
            s_code = e4m3_encode((amax16 / np.float32(E2M1_MAX) / gs).astype(np.float32))
        else:
            s_code = np.zeros(amax16.shape, dtype=np.uint8)
        s_val = e4m3_decode(s_code).astype(np.float32)
        denom = (s_val * gs).astype(np.float32)
        safe = np.where(denom > 0, denom, np.float32(1.0)).astype(np.float32)
        q = (xb / safe[..., None]).astype(np.float32)       # one correctly rounded fp32 division
        codes = np.where((denom > 0)[..., None], e2m1_encode(q), np.uint8(0)).astype(np.uint8).reshape(-1, K)
        packed[r0:r0 + chunk_rows] = pack_e2m1(codes)
        sf[r0:r0 + chunk_rows] = s_code
    return packed, sf


# ----------------------------------------------------------------------------- routing


def counts_to_indices(counts, order=None) -> np.ndarray:
    """Contiguous sorted runs: expert order[i] gets counts[order[i]] consecutive rows."""
    counts = np.asarray(counts, dtype=np.int64)
    G = counts.size
    order = np.arange(G) if order is None else np.asarray(order)
    parts = [np.full(int(counts[g]), g, dtype=np.int32) for g in order]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int32)


def run_starts(m_indices: np.ndarray):
    idx = np.asarray(m_indices)
    if idx.size == 0:
        return []
    starts = [0] + [int(i) for i in np.nonzero(idx[1:] != idx[:-1])[0] + 1]
    return starts


# ----------------------------------------------------------------------------- workloads


@dataclasses.dataclass
class Workload:
    name: str
    kind: str               # "fp8" or "nvfp4"
    M: int
    N: int
    K: int
    G: int
    A: np.ndarray            # fp8: uint8 [M,K]; nvfp4: uint8 [M,K/2]
    B: np.ndarray            # fp8: uint8 [G,N,K]; nvfp4: uint8 [G,N,K/2]
    m_indices: Optional[np.ndarray]   # int32 [M] or None (G == 1 only)
    a_scale: Optional[np.ndarray] = None   # fp8: f32 [M, K/128]
    b_scale: Optional[np.ndarray] = None   # fp8: f32 [G, ceil(N/128), K/128]
    sfa: Optional[np.ndarray] = None       # nvfp4: uint8 [M, K/16]
    sfb: Optional[np.ndarray] = None       # nvfp4: uint8 [G, N, K/16]
    alpha: Optional[np.ndarray] = None     # nvfp4: f32 [G]

    @property
    def routed_rows(self) -> int:
        if self.m_indices is None:
            return self.M
        idx = self.m_indices
        return int(np.count_nonzero((idx >= 0) & (idx < self.G)))

    @property
    def flops(self) -> float:
        return 2.0 * self.routed_rows * self.N * self.K

    def active_experts(self):
        if self.m_indices is None:
            return [0]
        idx = self.m_indices
        return sorted(set(int(g) for g in np.unique(idx) if 0 <= g < self.G))

    def algorithmic_bytes(self) -> int:
        """Compulsory traffic: A codes + A scales, B and its scales for active experts only,
        m_indices, alpha, and C in BF16 for routed rows."""
        act = len(self.active_experts())
        if self.kind == "fp8":
            nb = (self.N + 127) // 128
            kb = self.K // 128
            a = self.M * self.K + self.M * kb * 4
            b = act * (self.N * self.K + nb * kb * 4)
            extra = 0
        else:
            a = self.M * (self.K // 2) + self.M * (self.K // 16)
            b = act * (self.N * (self.K // 2) + self.N * (self.K // 16))
            extra = self.G * 4
        idx = 0 if self.m_indices is None else self.M * 4
        c = self.routed_rows * self.N * 2
        return int(a + b + extra + idx + c)


def _routing_rng(seed: int):
    _, _, r = np.random.SeedSequence(seed).spawn(3)
    return np.random.Generator(np.random.PCG64(r))


def _pool_map(fn, items):
    """Run ``fn`` over ``items`` on a thread pool (numpy releases the GIL in the heavy loops).
    Results are independent of the thread count: every chunk has its own spawned seed."""
    items = list(items)
    workers = max(1, min(len(items), os.cpu_count() or 1, 32))
    if workers == 1:
        return [fn(it) for it in items]
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        return list(ex.map(fn, items))


_ROW_CHUNK = 1024


def make_fp8(M, N, K, G, m_indices, seed, a_std=1.0, b_std=0.02, name="fp8"):
    ss_a, ss_b, _ = np.random.SeedSequence(seed).spawn(3)
    A = np.empty((M, K), dtype=np.uint8)
    a_scale = np.empty((M, K // 128), dtype=np.float32)
    chunks = list(range(0, M, _ROW_CHUNK))
    a_seeds = ss_a.spawn(len(chunks))

    def do_a(i):
        r0 = chunks[i]
        r1 = min(M, r0 + _ROW_CHUNK)
        rng = np.random.Generator(np.random.PCG64(a_seeds[i]))
        x = rng.standard_normal((r1 - r0, K), dtype=np.float32) * np.float32(a_std)
        A[r0:r1], a_scale[r0:r1] = quant_fp8_rows(x)

    _pool_map(do_a, range(len(chunks)))
    NB = (N + 127) // 128
    B = np.empty((G, N, K), dtype=np.uint8)
    b_scale = np.empty((G, NB, K // 128), dtype=np.float32)
    b_seeds = ss_b.spawn(G * NB)

    def do_b(j):
        g, nb = divmod(j, NB)
        n0, n1 = nb * 128, min(N, nb * 128 + 128)
        rng = np.random.Generator(np.random.PCG64(b_seeds[j]))
        w = rng.standard_normal((n1 - n0, K), dtype=np.float32) * np.float32(b_std)
        codes, s = quant_fp8_blocks(w)
        B[g, n0:n1] = codes
        b_scale[g, nb] = s[0]

    _pool_map(do_b, range(G * NB))
    idx = None if m_indices is None else np.ascontiguousarray(m_indices, dtype=np.int32)
    return Workload(name, "fp8", M, N, K, G, A, B, idx, a_scale=a_scale, b_scale=b_scale)


def make_nvfp4(M, N, K, G, m_indices, seed, name="nvfp4"):
    ss_a, ss_b, _ = np.random.SeedSequence(seed).spawn(3)

    def draw(seeds, rows, i, r0):
        rng = np.random.Generator(np.random.PCG64(seeds[i]))
        return rng.standard_normal((rows, K), dtype=np.float32)

    # The global scale needs the amax of the whole tensor, so each chunk is drawn twice (once for
    # the amax, once to quantise); drawing is cheap next to holding an fp32 copy of a large tensor.
    def quant_tensor(ss, R, out_codes, out_sf):
        chunks = list(range(0, R, _ROW_CHUNK))
        seeds = ss.spawn(len(chunks))
        amaxes = _pool_map(lambda i: float(np.abs(draw(seeds, min(R, chunks[i] + _ROW_CHUNK) - chunks[i],
                                                           i, chunks[i])).max()), range(len(chunks)))
        amax = np.float32(max(amaxes) if amaxes else 0.0)
        gs = np.float32(amax / np.float32(E4M3_MAX * E2M1_MAX))

        def do(i):
            r0 = chunks[i]
            r1 = min(R, r0 + _ROW_CHUNK)
            x = draw(seeds, r1 - r0, i, r0)
            out_codes[r0:r1], out_sf[r0:r1] = quant_nvfp4(x, gs)

        _pool_map(do, range(len(chunks)))
        return gs

    A = np.empty((M, K // 2), dtype=np.uint8)
    sfa = np.empty((M, K // 16), dtype=np.uint8)
    gsa = quant_tensor(ss_a, M, A, sfa)
    B = np.empty((G, N, K // 2), dtype=np.uint8)
    sfb = np.empty((G, N, K // 16), dtype=np.uint8)
    alpha = np.empty((G,), dtype=np.float32)
    b_seeds = ss_b.spawn(G)
    for g in range(G):
        gsb = quant_tensor(b_seeds[g], N, B[g], sfb[g])
        alpha[g] = np.float32(gsa * gsb)
    idx = None if m_indices is None else np.ascontiguousarray(m_indices, dtype=np.int32)
    return Workload(name, "nvfp4", M, N, K, G, A, B, idx, sfa=sfa, sfb=sfb, alpha=alpha)


def routing_multinomial_unaligned(M, G, rng, window=128, max_tries=10000):
    """Sorted contiguous runs with Multinomial(M, uniform) lengths, every count >= 1 and every run
    boundary off a multiple of the window (so runs start inside windows)."""
    for _ in range(max_tries):
        counts = rng.multinomial(M, [1.0 / G] * G)
        if counts.min() < 1:
            continue
        bounds = np.cumsum(counts)[:-1]
        if np.all(bounds % window != 0):
            return counts_to_indices(counts)
    raise RuntimeError("no admissible routing found")


def routing_uniform_cuts(M, G, rng, window=128, min_unaligned=None, max_tries=10000):
    """G runs from G-1 distinct uniform cut points in 1..M-1; at least half of the runs start off
    a window boundary."""
    need = (G + 1) // 2 if min_unaligned is None else min_unaligned
    for _ in range(max_tries):
        cuts = np.sort(rng.choice(np.arange(1, M), size=G - 1, replace=False))
        starts = np.concatenate([[0], cuts])
        if int(np.count_nonzero(starts % window != 0)) >= need:
            counts = np.diff(np.concatenate([starts, [M]]))
            return counts_to_indices(counts)
    raise RuntimeError("no admissible routing found")


def routing_zipf(M, G, rng, s=1.2):
    """Expert counts ~ Multinomial(M, p) with p_r proportional to r^-s over ranks r = 1..G, ranks
    mapped to experts by a seeded permutation; rows sorted by expert id."""
    ranks = np.arange(1, G + 1, dtype=np.float64)
    p = ranks ** (-s)
    p /= p.sum()
    perm = rng.permutation(G)
    p_expert = np.empty(G)
    p_expert[perm] = p
    counts = rng.multinomial(M, p_expert)
    return counts_to_indices(counts)


# The five benchmark workloads.  ``scale`` shrinks M (and N for the large ones) for quick tests
# while keeping the structure; scale=1 is the full size.


def config(i: int, seed: Optional[int] = None):
    seed = i if seed is None else seed
    rr = _routing_rng(seed)
    if i == 0:
        M, N, K, G = 512, 256, 512, 4
        idx = routing_multinomial_unaligned(M, G, rr)
        return make_fp8(M, N, K, G, idx, seed, name="fp8_g4_m512_n256_k512")
    if i == 1:
        M, N, K, G = 8192, 4096, 7168, 8
        idx = routing_uniform_cuts(M, G, rr)
        return make_fp8(M, N, K, G, idx, seed, name="fp8_moe_prefill_g8_m8192_n4096_k7168")
    if i == 2:
        M, N, K, G = 2048, 36864, 4608, 1
        return make_nvfp4(M, N, K, G, np.zeros(M, dtype=np.int32), seed,
                          name="nvfp4_dense_m2048_n36864_k4608")
    if i == 3:
        Mg, N, K, G = 8192, 8192, 8192, 8
        idx = counts_to_indices([Mg] * G)
        return make_nvfp4(Mg * G, N, K, G, idx, seed, name="nvfp4_grouped_g8_mg8192_n8192_k8192")
    if i == 4:
        M, N, K, G = 512, 4096, 7168, 64
        idx = routing_zipf(M, G, rr)
        return make_fp8(M, N, K, G, idx, seed, name="fp8_decode_zipf_g64_m512_n4096_k7168")
    raise ValueError(i)


CONFIG_NAMES = {
    0: "fp8_g4_m512_n256_k512",
    1: "fp8_moe_prefill_g8_m8192_n4096_k7168",
    2: "nvfp4_dense_m2048_n36864_k4608",
    3: "nvfp4_grouped_g8_mg8192_n8192_k8192",
    4: "fp8_decode_zipf_g64_m512_n4096_k7168",
}
