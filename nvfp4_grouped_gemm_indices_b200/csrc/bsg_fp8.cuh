// bsg_fp8.cuh -- FP8 (E4M3) grouped GEMM with FP32 per-128 block scales, BF16 out, sm_100a.
//
// Operation: the FP8 page ("[flashinfer] FlashInfer FP8 GEMM 최적화: 윈도우 세그먼트 KG1 프로그램으로
// GPU 성능 극대화", introduction and section 1):
//   C[m, n] = bf16( sum_kb a_scale[m, kb] * b_scale[g, n/128, kb] * (A[m, kb-block] . B[g, n, kb-block]) )
//
// Design (persistent, warp-specialised, one CTA per SM, 20 warps), templated on CG, the number of
// SMs one MMA spans:
//   CG = 1  a work unit is a 128-row window segment x 256 columns on one SM; two 256-column TMEM
//           accumulators ping-pong between the MMAs and the promotion.
//   CG = 2  a cluster of two CTAs on an SM pair computes a 256 x 256 tile with 2-SM tcgen05 MMAs
//           (cta_group::2): each CTA holds the 128 rows of its own window segment and 128 of the
//           256 B rows; the even CTA issues the MMAs for both.  Per SM and K block this moves 32 KB
//           of A/B through shared memory instead of 48 KB (the MMA reads each CTA's B half once for
//           both SMs); each CTA promotes its own 128 x 256 partials in two ping-pong accumulators.
// Roles:
//   warp 0      producer: TMA of the A box [128 rows x 128 B] and this CTA's B box [BN/CG rows x
//               128 B] into a STAGES-deep shared-memory ring; the arrival bytes of both CTAs of a
//               pair count on the even CTA's full barrier.
//   warp 1      TMEM allocator + (even CTA) single-thread tcgen05.mma issuer: per 128-K block, 4 K steps
//               of kind::f8f6f4 MMAs (128 x 256 per step, or 256 x 256 across the pair) into a fresh
//               FP32 accumulator; two 256-column accumulators ping-pong so the tensor cores run one
//               block ahead of the epilogue that promotes the previous block.  Completion is
//               committed to the barriers of both CTAs.
//   warp 2      scheduler (bsg_sched.cuh): window segmentation, pairing, unit hand-out.
//   warp 3      scale producer: cp.async of each K block's scales (a_scale of the 128 rows, b_scale
//               of the tile's 128-column blocks) into a separate, deeper scale ring that completes
//               on an mbarrier (cp.async.mbarrier.arrive).  Kept off the TMA producer's
//               sub-partition: there its scattered loads delayed the co-resident epilogue warps.
//   warps 4..19 epilogue (16 warps, 4 per SM sub-partition): warp w owns TMEM lanes 32*(w%4)..
//               (tile rows) and 64 columns; per K block it reads the fresh partial from TMEM and
//               accumulates partial * a_scale[row, kb] * b_scale[g, col/128, kb] into registers with
//               packed FP32x2 FMAs; after the last K block it rounds to BF16 and stores the rows of
//               its segment only.
// Pipeline state is one (stage, phase) pair per ring, advanced at every use and carried across work
// units; each acquire waits on the barrier right before the slot is written, so no token is held
// across a unit boundary (the failure mode the page "[cutlass] NVIDIA CUTLASS CuTeDSL: SM103 Grouped
// Block-Scaled GEMM 최적화 분석", section 2, fixed by resetting its producer per tile).
#pragma once

#include <cuda_bf16.h>

#include "bsg_ptx.cuh"
#include "bsg_sched.cuh"

namespace bsg {

struct Fp8Params {
  CUtensorMap tmA;  // uint8 [M, K]: dims {K, M}, box {128, 128}, 128B swizzle, rows zero-filled past M
  CUtensorMap tmB;  // uint8 [G, N, K]: dims {K, N, G}, box {128, 256/CG, 1}, 128B swizzle
  const float* a_scale;
  const float* b_scale;
  const int* m_indices;
  __nv_bfloat16* C;
  int M, N, K, G;
  int n_group;      // N tiles per raster group
  uint64_t timeout_ns;
  DeviceStatus* status;
  int debug_mode;
};

namespace fp8 {

constexpr int BM = 128;                 // rows per CTA
constexpr int BK = 128;                 // one scale block
constexpr int SC_STAGES = 12;           // scale ring: >= STAGES + ACC + slack
constexpr int Q = 4;                    // unit queue depth
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_SCHED = 2, WARP_SCALE = 3, WARP_EPI0 = 4;
constexpr int EPI_WARPS = 16;
constexpr int NUM_WARPS = WARP_EPI0 + EPI_WARPS;
constexpr int THREADS = NUM_WARPS * 32;
constexpr int TMEM_COLS = 512;

template <int CG, int BN_ = 256>
struct Cfg {
  static constexpr int BN = BN_;                          // output columns per unit: 256, or 64
  static constexpr int ACC = TMEM_COLS / BN;              // TMEM accumulators: 2 (256) or 8 (64)
  static constexpr int B_BOX_ROWS = BN / CG;              // B rows this CTA loads per stage
  static constexpr int A_BYTES = BM * BK;                 // 16 KB
  static constexpr int B_BYTES = B_BOX_ROWS * BK;         // 32 KB (CG 1) / 16 KB (CG 2) / 8 KB (64)
  static constexpr int STAGES = BN == 64 ? 8 : (CG == 1 ? 4 : 6);   // 192 KB of ring in each case
  static constexpr uint32_t STAGE_TX = CG * (A_BYTES + B_BYTES);  // bytes counted on the even CTA
  static constexpr int EPI_COLS = BN / 4;                 // columns per epilogue warp: 64 or 16
  static constexpr int NB_TILE = BN >= 128 ? BN / 128 : 1;  // 128-column scale blocks per tile
};

struct ScaleSlot {
  float a[BM];         // a_scale[row0 + r, kb]
  float b[2];          // b_scale[g, n0/128 + h, kb], h < NB_TILE
  float pad[2];
};

template <int CG, int BN = 256>
struct alignas(1024) Smem {
  uint8_t a[Cfg<CG, BN>::STAGES][Cfg<CG, BN>::A_BYTES];
  uint8_t b[Cfg<CG, BN>::STAGES][Cfg<CG, BN>::B_BYTES];
  ScaleSlot sc[SC_STAGES];
  uint64_t full[Cfg<CG, BN>::STAGES];   // CG 1: own loads; CG 2: (even CTA) both CTAs' loads
  uint64_t empty[Cfg<CG, BN>::STAGES];  // one MMA commit (multicast to both CTAs of a pair)
  uint64_t sc_full[SC_STAGES];      // 32 cp.async arrivals (one per producer lane)
  uint64_t sc_empty[SC_STAGES];     // EPI_WARPS arrivals
  uint64_t tmem_full[Cfg<CG, BN>::ACC];   // one MMA commit
  uint64_t tmem_empty[Cfg<CG, BN>::ACC];  // (even CTA) CG * EPI_WARPS arrivals
  uint64_t mma_done;
  UnitQueue<Q> queue;
  uint32_t tmem_base;
  int abort;
};

template <int CG, int BN = 256>
constexpr size_t smem_bytes() {
  return sizeof(Smem<CG, BN>) + 1024;  // + alignment slack
}

template <int CG, int BN = 256>
__device__ __forceinline__ Smem<CG, BN>& smem_ref(uint8_t* raw) {
  uintptr_t p = reinterpret_cast<uintptr_t>(raw);
  p = (p + 1023) & ~static_cast<uintptr_t>(1023);
  return *reinterpret_cast<Smem<CG, BN>*>(p);
}

// 4-byte cp.async global -> shared; src_bytes = 0 zero-fills the destination without reading.
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "r"(src_bytes)
               : "memory");
}

// The mbarrier receives one arrival once all of this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int CG, int BN_ = 256>
__device__ __forceinline__ void fp8_kernel_body(const Fp8Params& p) {
  using C = Cfg<CG, BN_>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  Smem<CG, BN_>& s = smem_ref<CG, BN_>(smem_raw);
  const int warp = warp_idx();
  const int lane = lane_idx();
  const int KB = p.K / BK;
  constexpr int BN = C::BN;
  constexpr int ACC = C::ACC;
  constexpr int EPI_COLS = C::EPI_COLS;
  const int n_tiles = (p.N + BN - 1) / BN;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;   // 0 = the CTA that issues the MMAs
  WaitCtx wctx{p.timeout_ns, &s.abort, p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < SC_STAGES; ++i) {
      mbar_init(&s.sc_full[i], 32);
      mbar_init(&s.sc_empty[i], EPI_WARPS);
    }
    for (int i = 0; i < C::ACC; ++i) {
      mbar_init(&s.tmem_full[i], 1);
      mbar_init(&s.tmem_empty[i], CG * EPI_WARPS);
    }
    for (int i = 0; i < Q; ++i) {
      mbar_init(&s.queue.full[i], 1);
      mbar_init(&s.queue.empty[i], EPI_WARPS + 3);
    }
    mbar_init(&s.mma_done, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
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
  } else if (warp == WARP_SCALE) {
    // scale producer: the K block's a_scale (128 rows of the window) and b_scale (the tile's
    // 128-column blocks) by cp.async into the scale ring; a warp of its own keeps these scattered
    // 4-byte loads off the sub-partition of the TMA producer
    const int NB = (p.N + 127) / 128;
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<SC_STAGES> spos;
    long long issued = 0;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx)) {
        ok = false;
        break;
      }
      if (!u.valid) break;
      const int nb0 = u.n0 / 128;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.sc_empty[spos.stage], spos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteSmemEmpty, 16 + spos.stage)) {
          ok = false;
          break;
        }
        ScaleSlot& slot = s.sc[spos.stage];
#pragma unroll
        for (int i = 0; i < BM / 32; ++i) {
          const int row = u.row0 + i * 32 + lane;
          const bool in = row < p.M;
          cp_async_4(&slot.a[i * 32 + lane], p.a_scale + static_cast<size_t>(in ? row : 0) * KB + kb, in ? 4u : 0u);
        }
        if (lane < C::NB_TILE) {
          const bool in = nb0 + lane < NB;
          cp_async_4(&slot.b[lane], p.b_scale + (static_cast<size_t>(u.g) * NB + (in ? nb0 + lane : 0)) * KB + kb,
                     in ? 4u : 0u);
        }
        cp_async_arrive(&s.sc_full[spos.stage]);
        ++issued;
        spos.advance();
      }
    }
    if (!ok) drain_inflight_loads<SC_STAGES>(s.sc_full, spos, issued, wctx);
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
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.empty[pos.stage], pos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteSmemEmpty, pos.stage)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          // this CTA's B box: rows n0 + rank * B_BOX_ROWS of expert g
          if (CG == 1) {
            mbar_arrive_expect_tx(&s.full[pos.stage], C::STAGE_TX);
            tma_load_2d(s.a[pos.stage], &p.tmA, &s.full[pos.stage], kb * BK, u.row0);
            tma_load_3d(s.b[pos.stage], &p.tmB, &s.full[pos.stage], kb * BK, u.n0, u.g);
          } else {
            const uint32_t leader_full = mapa_shared(smem_u32(&s.full[pos.stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&s.full[pos.stage], C::STAGE_TX);
            tma_load_2d_pair(s.a[pos.stage], &p.tmA, leader_full, kb * BK, u.row0);
            tma_load_3d_pair(s.b[pos.stage], &p.tmB, leader_full, kb * BK,
                             u.n0 + static_cast<int>(rank) * C::B_BOX_ROWS, u.g);
          }
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
      // (CG 2: the odd CTA's loads land on the even CTA's barrier; the closing cluster barrier keeps
      // this CTA's shared memory alive until the even CTA has drained those too.)
      if (CG == 1 || rank == 0) drain_inflight_loads<STAGES>(s.full, pos, issued, wctx);
    }
  } else if (warp == WARP_MMA) {
    constexpr uint32_t IDESC = idesc_f8f6f4_e4m3(BM * CG, BN);
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    RingPos<ACC> accp;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      if (CG == 2 && rank != 0) continue;  // the even CTA issues the pair's MMAs
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.full[pos.stage], pos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSmemFull,
                       pos.stage)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&s.tmem_empty[accp.stage], accp.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteTmemEmpty, accp.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = sdesc_k_sw128(smem_u32(s.a[pos.stage]));
          const uint64_t db = sdesc_k_sw128(smem_u32(s.b[pos.stage]));
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(accp.stage * BN);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            // +32 bytes of K per step inside the 128-byte swizzled row (2 x 16-byte units)
            if (CG == 1)
              mma_f8f6f4(d_tmem, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k), IDESC,
                         k > 0 ? 1u : 0u);
            else
              mma_f8f6f4_pair(d_tmem, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k), IDESC,
                              k > 0 ? 1u : 0u);
          }
          if (CG == 1) {
            tc_commit(&s.empty[pos.stage]);
            tc_commit(&s.tmem_full[accp.stage]);
          } else {
            tc_commit_pair_multicast(&s.empty[pos.stage], 0x3);
            tc_commit_pair_multicast(&s.tmem_full[accp.stage], 0x3);
          }
        }
        __syncwarp();
        pos.advance();
        accp.advance();
      }
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
  } else if (warp >= WARP_EPI0) {
    // ------------------------------------------------------------------ epilogue warps
    const int quarter = warp & 3;                      // TMEM lane quarter this warp may access
    const int cg = (warp - WARP_EPI0) >> 2;            // column group of the tile (4 groups)
    const int r = quarter * 32 + lane;                 // tile row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int h = (cg * EPI_COLS) / 128;               // which 128-column scale block
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<ACC> accp;
    RingPos<SC_STAGES> spos;
    while (true) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      float2 accum[EPI_COLS / 2];
#pragma unroll
      for (int i = 0; i < EPI_COLS / 2; ++i) accum[i] = make_float2(0.f, 0.f);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.sc_full[spos.stage], spos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteTmemFull,
                       16 + spos.stage)) {
          ok = false;
          break;
        }
        const float sv = s.sc[spos.stage].a[r] * s.sc[spos.stage].b[h];
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.sc_empty[spos.stage]);
        spos.advance();
        const float2 scale = make_float2(sv, sv);
        if (!mbar_wait(&s.tmem_full[accp.stage], accp.phase, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteTmemFull, accp.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + static_cast<uint32_t>(accp.stage * BN + cg * EPI_COLS);
        if constexpr (EPI_COLS % 32 == 0) {
#pragma unroll
          for (int c = 0; c < EPI_COLS; c += 32) {
            uint32_t v0[16], v1[16];
            tmem_ld_x16(taddr + c, v0);
            tmem_ld_x16(taddr + c + 16, v1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              accum[c / 2 + i] = __ffma2_rn(make_float2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1])),
                                            scale, accum[c / 2 + i]);
              accum[c / 2 + 8 + i] = __ffma2_rn(
                  make_float2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1])), scale, accum[c / 2 + 8 + i]);
            }
          }
        } else {                                         // 16 columns per warp (the 64-column tile)
          uint32_t v0[16];
          tmem_ld_x16(taddr, v0);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            accum[i] = __ffma2_rn(make_float2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1])), scale,
                                  accum[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 1)
            mbar_arrive(&s.tmem_empty[accp.stage]);
          else
            mbar_arrive_cluster(mapa_shared(smem_u32(&s.tmem_empty[accp.stage]), 0));
        }
        accp.advance();
      }
      if (!ok) break;
      // masked BF16 store of this thread's row: only rows of the segment, only columns < N
      const int row = u.row0 + r;
      const int col0 = u.n0 + cg * EPI_COLS;
      if (row >= u.row_lo && row < u.row_hi && col0 < p.N) {
        const int ncols = min(EPI_COLS, p.N - col0);
        __nv_bfloat16* dst = p.C + static_cast<size_t>(row) * p.N + col0;
#pragma unroll
        for (int c = 0; c < EPI_COLS; c += 8) {
          if (c < ncols) {
            uint4 v;
            v.x = pack_bf16x2(accum[c / 2 + 0].x, accum[c / 2 + 0].y);
            v.y = pack_bf16x2(accum[c / 2 + 1].x, accum[c / 2 + 1].y);
            v.z = pack_bf16x2(accum[c / 2 + 2].x, accum[c / 2 + 2].y);
            v.w = pack_bf16x2(accum[c / 2 + 3].x, accum[c / 2 + 3].y);
            *reinterpret_cast<uint4*>(dst + c) = v;
          }
        }
      }
    }
  }

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

__global__ void __launch_bounds__(THREADS, 1) bsg_fp8_grouped_kernel(const __grid_constant__ Fp8Params p) {
  fp8_kernel_body<1>(p);
}

// Launched as clusters of 2 CTAs (grid a multiple of 2).
__global__ void __launch_bounds__(THREADS, 1) bsg_fp8_grouped_2sm_kernel(const __grid_constant__ Fp8Params p) {
  fp8_kernel_body<2>(p);
}

// The 64-column tile for small problems: four times as many units as the 256-column tile, each a
// quarter of the MMA, promotion and store work per K block, eight accumulators and an eight-stage
// ring; on a grid that does not fill the GPU its units finish sooner.
__global__ void __launch_bounds__(THREADS, 1) bsg_fp8_grouped_n64_kernel(const __grid_constant__ Fp8Params p) {
  fp8_kernel_body<1, 64>(p);
}

}  // namespace fp8
}  // namespace bsg
