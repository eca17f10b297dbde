// bsg_nvfp4.cuh -- NVFP4 (E2M1 + UE4M3 per-16 scales + FP32 alpha) grouped GEMM, BF16 out, sm_100a.
//
// Operation: the native FP4 x FP4 grouped GEMM of the page "[onnxruntime] ONNX Runtime: Blackwell
// (SM120+)에서 NVFP4 QMoE를 위한 네이티브 FP4xFP4 Prefill 최적화", section 1:
//   C[m, n] = bf16( alpha[g] * sum_j sfa[m, j] * sfb[g, n, j] * (A[m, block j] . B[g, n, block j]) )
//
// Design (persistent, warp-specialised, one CTA per SM), templated on CG, the number of SMs one MMA
// spans:
//   CG = 1  a work unit is a 128-row window segment x 256 columns on one SM.
//   CG = 2  a cluster of two CTAs on an SM pair computes a 256 x 256 tile with 2-SM MMAs
//           (cta_group::2): each CTA holds the 128 rows of its own window segment and 128 of the 256
//           B rows (so each SM moves 32 KB of A/B per stage through shared memory instead of 48 KB)
//           and its own scale slots (SFA of its rows, SFB of all 256 columns); the even CTA issues
//           the MMAs and commits to both CTAs' barriers.
//   warps 0..7   epilogue: after the last K stage of a unit, read the 128 x BN FP32 accumulator from
//                TMEM (warp w: lanes 32*(w%4).., columns 128*(w/4)..), scale by alpha[g] and pack to
//                BF16 while reading, release the accumulator, then store the segment's rows: in the
//                pair kernel, when all 128 rows of the CTA belong to the segment, through a per-warp
//                128B-swizzled staging tile and TMA stores (2 x 32 rows x 64 columns); otherwise, and
//                in the one-SM kernel (no shared memory left beside its ring), with masked 16-byte
//                register stores.
//   warp 8       TMA producer for A and B (K stage = 256 elements = 128 packed bytes, 128B swizzle);
//                it also loads the stage's row-major scale bytes (sfa: 128 rows x 16 B, sfb: BN rows
//                x 16 B) with TMA into a raw per-stage buffer.
//   warp 9       TMEM allocator + single-thread issuer: per K stage, 4 x (128 x BN x 64)
//                kind::mxf4nvf4 block16 MMAs accumulating the whole K in one TMEM accumulator, the
//                scale factors read from the stage's TMEM scale slot (hardware block scaling).
//   warp 10      scheduler (bsg_sched.cuh).
//   warps 11..14 scale-factor writers, one per SM sub-partition (warp % 4 = TMEM lane quarter):
//                read the stage's raw scale bytes from shared memory into registers, rearrange them
//                and write them with tcgen05.st into the stage's TMEM scale slot, then arrive on the
//                stage's `full` barrier next to the TMA bytes.  Separate scale-factor warps follow
//                the warp-role split of the page "[cutlass] NVIDIA CUTLASS CuTeDSL: SM103 Grouped
//                Block-Scaled GEMM 최적화 분석", section 1.  Writing TMEM from registers keeps the
//                scale copies off the tensor pipe: a tcgen05.cp occupies the tensor pipe for about a
//                third of an MMA's time and does not overlap the MMAs (12 per stage cost ~70% of the
//                stage's MMA time when measured alone).
// TMEM columns: [0, BN) accumulator; scale slot s (one per pipeline stage) at 256 + 48 s: SFA in
// 16 columns (4 per 64-K MMA step), SFB in 32 columns (8 per step).  A step's scales are replicated
// in all four lane quarters: lane 32q + l, column c of SFA holds the 4 scales of row 32c + l; SFB
// column c holds those of row 32c + l (c < 8).  Each scale warp writes its own quarter.
#pragma once

#include <cuda_bf16.h>

#include "bsg_ptx.cuh"
#include "bsg_sched.cuh"

namespace bsg {

struct Nvfp4Params {
  CUtensorMap tmA;  // uint8 [M, K/2]:    dims {K/2, M},    box {128, 128},  128B swizzle
  CUtensorMap tmB;  // uint8 [G, N, K/2]: dims {K/2, N, G}, box {128, BN, 1}, 128B swizzle
  CUtensorMap tmSFA;  // uint8 [M, K/16]:    dims {K/16, M},    box {16, 128}
  CUtensorMap tmSFB;  // uint8 [G, N, K/16]: dims {K/16, N, G}, box {16, BN, 1}
  CUtensorMap tmC;    // bf16 C as bytes [M, 2N]: dims {2N, M}, box {128, 32}, 128B swizzle
  const float* alpha;
  const int* m_indices;
  __nv_bfloat16* C;
  int M, N, K, G;
  int n_group;        // N tiles per raster group
  uint64_t timeout_ns;
  DeviceStatus* status;
  int debug_mode;
};

namespace nvfp4 {

// TMA store of a tile from shared memory (bulk-group completion) and its helpers (the C epilogue of
// the pair kernel).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

constexpr int BM = 128;                  // rows per CTA
constexpr int BN = 256;                  // output columns per unit (both variants)
constexpr int BK = 256;                  // K elements per stage (128 packed bytes)
constexpr int Q = 4;
constexpr int EPI_WARPS = 8;
constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_SCHED = 10, WARP_SF0 = 11;
constexpr int SF_WARPS = 4;
constexpr int NUM_WARPS = WARP_SF0 + SF_WARPS;
constexpr int THREADS = NUM_WARPS * 32;
constexpr int A_BYTES = BM * BK / 2;     // 16 KB
constexpr int SFA_BYTES = BM * BK / 16;  // 2 KB
constexpr int SFB_BYTES = BN * BK / 16;  // 4 KB (every CTA holds the scales of all BN columns)
constexpr int TMEM_COLS = 512;
constexpr uint32_t COL_SF0 = 256;        // first scale slot
constexpr uint32_t SF_SLOT_COLS = 48;    // 16 SFA + 32 SFB columns per stage
constexpr uint32_t SFB_OFF = 16;

template <int CG>
struct Cfg {
  static constexpr int B_BOX_ROWS = BN / CG;                       // B rows this CTA loads per stage
  static constexpr int B_BYTES = B_BOX_ROWS * BK / 2;              // 32 KB (CG 1) / 16 KB (CG 2)
  static constexpr int STAGES = CG == 1 ? 4 : 5;                   // 216 KB / 190 KB of ring
  static constexpr uint32_t STAGE_TX = CG * (A_BYTES + B_BYTES);   // A/B bytes counted on the even CTA
  static constexpr int FULL_ARRIVALS = 1 + CG * SF_WARPS;          // TMA warp + every CTA's scale warps
  static_assert(COL_SF0 + STAGES * SF_SLOT_COLS <= TMEM_COLS, "scale slots exceed TMEM");
};

template <int CG>
struct alignas(1024) Smem {
  uint8_t a[Cfg<CG>::STAGES][A_BYTES];
  uint8_t b[Cfg<CG>::STAGES][Cfg<CG>::B_BYTES];
  alignas(128) uint8_t sf[Cfg<CG>::STAGES][SFA_BYTES + SFB_BYTES];  // raw row-major scale bytes (TMA)
  // (pair kernel) each epilogue warp's C staging tile: 32 rows x 64 BF16, 128B-swizzled for the TMA store
  alignas(1024) uint8_t stage_c[CG == 2 ? EPI_WARPS : 1][CG == 2 ? 32 * 128 : 16];
  uint64_t full[Cfg<CG>::STAGES];    // (even CTA) A/B bytes + FULL_ARRIVALS arrivals
  uint64_t sf_raw[Cfg<CG>::STAGES];  // this CTA's raw scale bytes landed (1 arrival + bytes)
  uint64_t empty[Cfg<CG>::STAGES];   // 1 MMA commit: the stage's smem and TMEM scale slot are free
  uint64_t tmem_full;
  uint64_t tmem_empty;               // (even CTA) CG * EPI_WARPS arrivals
  uint64_t mma_done;
  UnitQueue<Q> queue;
  uint32_t tmem_base;
  int abort;
};

template <int CG>
constexpr size_t smem_bytes() {
  return sizeof(Smem<CG>) + 1024;  // + alignment slack
}
static_assert(smem_bytes<1>() <= 232448 && smem_bytes<2>() <= 232448, "nvfp4 kernels' shared memory above 227 KB");

template <int CG>
__device__ __forceinline__ Smem<CG>& smem_ref(uint8_t* raw) {
  uintptr_t p = reinterpret_cast<uintptr_t>(raw);
  p = (p + 1023) & ~static_cast<uintptr_t>(1023);
  return *reinterpret_cast<Smem<CG>*>(p);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int k) {
  return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

template <int CG>
__device__ __forceinline__ void nvfp4_kernel_body(const Nvfp4Params& p) {
  using C = Cfg<CG>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  Smem<CG>& s = smem_ref<CG>(smem_raw);
  const int warp = warp_idx();
  const int lane = lane_idx();
  const int KS = p.K / BK;
  const int n_tiles = (p.N + BN - 1) / BN;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;   // 0 = the CTA that issues the MMAs
  WaitCtx wctx{p.timeout_ns, &s.abort, p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], C::FULL_ARRIVALS);
      mbar_init(&s.empty[i], 1);
      mbar_init(&s.sf_raw[i], 1);
    }
    mbar_init(&s.mma_done, 1);
    mbar_init(&s.tmem_full, 1);
    mbar_init(&s.tmem_empty, CG * EPI_WARPS);
    for (int i = 0; i < Q; ++i) {
      mbar_init(&s.queue.full[i], 1);
      mbar_init(&s.queue.empty[i], EPI_WARPS + 2 + SF_WARPS);
    }
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
    tma_prefetch_desc(&p.tmSFA);
    tma_prefetch_desc(&p.tmSFB);
  }
  if (warp == WARP_MMA) {
    if (CG == 2) {
      tmem_alloc_pair(&s.tmem_base, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&s.tmem_base, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (CG == 2) {
    cluster_sync();  // both CTAs' barriers are initialised before either touches the other's
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  // Small launches run as programmatic dependents of the previous kernel on the stream: the set-up
  // above overlapped it; wait for it to complete (its writes visible) before touching global memory,
  // then let the next kernel start its own set-up.  Without that launch attribute both are no-ops.
  grid_dependency_wait();
  grid_dependents_launch();

  if (warp == WARP_SCHED) {
    run_scheduler<Q, BN, CG == 2>(s.queue, p.m_indices, p.M, p.G, n_tiles, p.n_group, wctx, p.debug_mode);
  } else if (warp == WARP_TMA) {
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    long long issued = 0;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx)) {
        ok = false;
        break;
      }
      if (!u.valid) break;
      for (int kb = 0; kb < KS; ++kb) {
        if (!mbar_wait(&s.empty[pos.stage], pos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteSmemEmpty, pos.stage)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          if (CG == 1) {
            mbar_arrive_expect_tx(&s.full[pos.stage], C::STAGE_TX);
            tma_load_2d(s.a[pos.stage], &p.tmA, &s.full[pos.stage], kb * (BK / 2), u.row0);
            tma_load_3d(s.b[pos.stage], &p.tmB, &s.full[pos.stage], kb * (BK / 2), u.n0, u.g);
          } else {
            // A/B bytes of both CTAs count on the even CTA's full barrier; this CTA's B box is rows
            // n0 + rank * 128 of expert g
            const uint32_t leader_full = mapa_shared(smem_u32(&s.full[pos.stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&s.full[pos.stage], C::STAGE_TX);
            tma_load_2d_pair(s.a[pos.stage], &p.tmA, leader_full, kb * (BK / 2), u.row0);
            tma_load_3d_pair(s.b[pos.stage], &p.tmB, leader_full, kb * (BK / 2),
                             u.n0 + static_cast<int>(rank) * C::B_BOX_ROWS, u.g);
          }
          // this CTA's own scale bytes (SFA of its rows, SFB of all BN columns) on its own barrier
          mbar_arrive_expect_tx(&s.sf_raw[pos.stage], SFA_BYTES + SFB_BYTES);
          tma_load_2d(s.sf[pos.stage], &p.tmSFA, &s.sf_raw[pos.stage], kb * (BK / 16), u.row0);
          tma_load_3d(s.sf[pos.stage] + SFA_BYTES, &p.tmSFB, &s.sf_raw[pos.stage], kb * (BK / 16), u.n0, u.g);
        }
        __syncwarp();
        ++issued;
        pos.advance();
      }
    }
    if (ok) {
      // producer tail: every stage handed out has been consumed before the CTA may retire
      for (int i = 0; i < STAGES; ++i) {
        if (!mbar_wait(&s.empty[pos.stage], pos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status, kSiteDrain,
                       pos.stage))
          break;
        pos.advance();
      }
    } else {
      // (CG 2: the odd CTA's A/B loads land on the even CTA's barrier; the closing cluster barrier
      // keeps this CTA's shared memory alive until the even CTA has drained those too.)
      if (CG == 1 || rank == 0) drain_inflight_loads<STAGES>(s.full, pos, issued, wctx);
      drain_inflight_loads<STAGES>(s.sf_raw, pos, issued, wctx);
    }
  } else if (warp >= WARP_SF0) {
    // ------------------------------------------------------------------ scale-factor warps
    // Every quarter receives the same words (the replicated layout): lane l reads raw rows l + 32c.
    const int qt = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(qt * 32) << 16;
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx)) break;
      if (!u.valid) break;
      for (int kb = 0; kb < KS; ++kb) {
        // the raw bytes of this use of the stage have landed (they were loaded after the stage was
        // freed, so the slot's previous MMAs are complete as well)
        if (!mbar_wait(&s.sf_raw[pos.stage], pos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSfRaw,
                       pos.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint4* raw = reinterpret_cast<const uint4*>(s.sf[pos.stage]);
        uint4 va[4], vb[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) va[c] = raw[32 * c + lane];
#pragma unroll
        for (int c = 0; c < 8; ++c) vb[c] = raw[BM + 32 * c + lane];
        uint32_t ra16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) ra16[j] = word(va[j & 3], j >> 2);
        uint32_t rb32[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) rb32[j] = word(vb[j & 7], j >> 3);
        const uint32_t slot = tmem_base + lane_addr + COL_SF0 + static_cast<uint32_t>(pos.stage) * SF_SLOT_COLS;
        tmem_st_x16(slot, ra16);
        tmem_st_x32(slot + SFB_OFF, rb32);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 1 || rank == 0)
            mbar_arrive(&s.full[pos.stage]);
          else
            mbar_arrive_cluster(mapa_shared(smem_u32(&s.full[pos.stage]), 0));
        }
        pos.advance();
      }
    }
  } else if (warp == WARP_MMA) {
    constexpr uint32_t IDESC = idesc_mxf4nvf4(BM * CG, BN);
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    uint32_t acc_phase = 0;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      if (CG == 2 && rank != 0) continue;  // the even CTA issues the pair's MMAs
      if (!mbar_wait(&s.tmem_empty, acc_phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status, kSiteTmemEmpty, 0))
        break;
      tc_fence_after();
      for (int kb = 0; kb < KS; ++kb) {
        if (!mbar_wait(&s.full[pos.stage], pos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSmemFull,
                       pos.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = sdesc_k_sw128(smem_u32(s.a[pos.stage]));
          const uint64_t db = sdesc_k_sw128(smem_u32(s.b[pos.stage]));
          const uint32_t sf = tmem_base + COL_SF0 + static_cast<uint32_t>(pos.stage) * SF_SLOT_COLS;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            if (CG == 1)
              mma_mxf4nvf4(tmem_base, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k), IDESC,
                           sf + 4 * k, sf + SFB_OFF + 8 * k, acc);
            else
              mma_mxf4nvf4_pair(tmem_base, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k),
                                IDESC, sf + 4 * k, sf + SFB_OFF + 8 * k, acc);
          }
          if (CG == 1) {
            tc_commit(&s.empty[pos.stage]);
            if (kb == KS - 1) tc_commit(&s.tmem_full);
          } else {
            tc_commit_pair_multicast(&s.empty[pos.stage], 0x3);
            if (kb == KS - 1) tc_commit_pair_multicast(&s.tmem_full, 0x3);
          }
        }
        __syncwarp();
        pos.advance();
      }
      acc_phase ^= 1u;
    }
    // every MMA this thread issued has completed before TMEM may be released
    if (CG == 1 || rank == 0) {
      if (lane == 0) {
        if (CG == 1)
          tc_commit(&s.mma_done);
        else
          tc_commit_pair_multicast(&s.mma_done, 0x1);
      }
      __syncwarp();
      mbar_wait(&s.mma_done, 0, wctx.timeout_ns, nullptr, nullptr, kSiteDrain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps 0..7
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int qslot = 0;
    uint32_t qphase = 0;
    uint32_t acc_phase = 0;
    while (true) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      const float alpha = __ldg(p.alpha + u.g);
      if (!mbar_wait(&s.tmem_full, acc_phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteTmemFull, 0)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + lane_addr + static_cast<uint32_t>(half * 128);
      uint32_t o[64];  // 128 BF16 values of this row, packed in pairs
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        uint32_t v0[16], v1[16];
        tmem_ld_x16(taddr + c, v0);
        tmem_ld_x16(taddr + c + 16, v1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[c / 2 + i] = pack_bf16x2(__uint_as_float(v0[2 * i]) * alpha, __uint_as_float(v0[2 * i + 1]) * alpha);
          o[c / 2 + 8 + i] =
              pack_bf16x2(__uint_as_float(v1[2 * i]) * alpha, __uint_as_float(v1[2 * i + 1]) * alpha);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 1 || rank == 0)
          mbar_arrive(&s.tmem_empty);
        else
          mbar_arrive_cluster(mapa_shared(smem_u32(&s.tmem_empty), 0));
      }
      acc_phase ^= 1u;
      const int row = u.row0 + r;
      const int col0 = u.n0 + half * 128;
      if (CG == 2 && u.row_lo <= u.row0 && u.row_hi >= u.row0 + BM && col0 < p.N) {
        // every row of this CTA belongs to the unit's segment: two TMA stores of 32 rows x 64 columns
        // per warp through a 128B-swizzled staging tile (columns past N are clipped by the store)
        const uint32_t sbase = smem_u32(s.stage_c[warp]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (col0 + 64 * c >= p.N) break;               // warp-uniform: the chunk lies past N
          if (lane == 0) bulk_wait_read0();            // the previous store has read the tile
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(sbase + lane * 128 + ((j ^ (lane & 7)) << 4), o[32 * c + 4 * j], o[32 * c + 4 * j + 1],
                         o[32 * c + 4 * j + 2], o[32 * c + 4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&p.tmC, s.stage_c[warp], (col0 + 64 * c) * 2, u.row0 + quarter * 32);
            bulk_commit();
          }
        }
      } else if (row >= u.row_lo && row < u.row_hi && col0 < p.N) {
        const int ncols = min(128, p.N - col0);
        __nv_bfloat16* dst = p.C + static_cast<size_t>(row) * p.N + col0;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          if (c < ncols)
            *reinterpret_cast<uint4*>(dst + c) = make_uint4(o[c / 2], o[c / 2 + 1], o[c / 2 + 2], o[c / 2 + 3]);
        }
      }
    }
  }

  if (CG == 2 && warp < EPI_WARPS && lane == 0) bulk_wait0();   // this warp's TMA stores are complete
  tc_fence_before();
  if (CG == 2) {
    cluster_sync();  // the even CTA's MMAs into the odd CTA's TMEM are complete (mma_done waited)
  } else {
    __syncthreads();
  }
  tc_fence_after();
  if (warp == WARP_MMA) {
    if (CG == 2)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

__global__ void __launch_bounds__(THREADS, 1) bsg_nvfp4_grouped_kernel(const __grid_constant__ Nvfp4Params p) {
  nvfp4_kernel_body<1>(p);
}

// Launched as clusters of 2 CTAs (grid a multiple of 2).
__global__ void __launch_bounds__(THREADS, 1) bsg_nvfp4_grouped_2sm_kernel(const __grid_constant__ Nvfp4Params p) {
  nvfp4_kernel_body<2>(p);
}

}  // namespace nvfp4
}  // namespace bsg
