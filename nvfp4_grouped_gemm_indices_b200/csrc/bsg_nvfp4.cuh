// bsg_nvfp4.cuh -- NVFP4 (E2M1 + UE4M3 per-16 scales + FP32 alpha) grouped GEMM, BF16 out, sm_100a.
//
// Operation: the native FP4 x FP4 grouped GEMM of the page "[onnxruntime] ONNX Runtime: Blackwell
// (SM120+)에서 NVFP4 QMoE를 위한 네이티브 FP4xFP4 Prefill 최적화", section 1:
//   C[m, n] = bf16( alpha[g] * sum_j sfa[m, j] * sfb[g, n, j] * (A[m, block j] . B[g, n, block j]) )
//
// Design (persistent, warp-specialised, one CTA per SM; same skeleton as the FP8 kernel):
//   warps 0..7  epilogue: after the last K stage of a unit, read the 128 x BN FP32 accumulator from
//               TMEM (warp w: lanes 32*(w%4).., columns 128*(w/4)..), release it, multiply by
//               alpha[g], round to BF16, store the segment's rows.
//   warp 8      TMA producer for A and B (K stage = 256 elements = 128 packed bytes, 128B swizzle).
//   warp 9      TMEM allocator + single-thread issuer: per K stage, tcgen05.cp of the stage's scale
//               factors into TMEM, then 4 x (128 x BN x 64) kind::mxf4nvf4 block16 MMAs accumulating
//               the whole K in one TMEM accumulator (hardware block scaling).
//   warp 10     scheduler (bsg_sched.cuh).
//   warp 11     scale-factor producer: TMA of the row-major scale bytes of the stage (sfa: 128 rows x
//               16 B, sfb: BN rows x 16 B) and an in-place shuffle into the layout tcgen05.cp takes
//               (for each 64-K MMA step, 32 rows of 16 B each holding rows r, r+32, r+64, r+96),
//               then a fence to the async proxy and an arrival on the stage's sf_full barrier.  A
//               separate warp for the scale factors follows the warp-role split of the page
//               "[cutlass] NVIDIA CUTLASS CuTeDSL: SM103 Grouped Block-Scaled GEMM 최적화 분석",
//               section 1.
// TMEM columns: [0, BN) accumulator, [256, 272) SFA (4 columns per MMA step), [272, 304) SFB
// (8 columns per MMA step for BN = 256).
#pragma once

#include <cuda_bf16.h>

#include "bsg_ptx.cuh"
#include "bsg_sched.cuh"

namespace bsg {

struct Nvfp4Params {
  CUtensorMap tmA;    // uint8 [M, K/2]:   dims {K/2, M},     box {128, 128},  128B swizzle
  CUtensorMap tmB;    // uint8 [G, N, K/2]: dims {K/2, N, G}, box {128, BN, 1}, 128B swizzle
  CUtensorMap tmSFA;  // uint8 [M, K/16]:  dims {K/16, M},    box {16, 128}
  CUtensorMap tmSFB;  // uint8 [G, N, K/16]: dims {K/16, N, G}, box {16, BN, 1}
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

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                  // K elements per stage (128 packed bytes)
constexpr int STAGES = 4;
constexpr int Q = 4;
constexpr int EPI_WARPS = 8;
constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_SCHED = 10, WARP_SF = 11;
constexpr int NUM_WARPS = 12;
constexpr int THREADS = NUM_WARPS * 32;
constexpr int A_BYTES = BM * BK / 2;     // 16 KB
constexpr int B_BYTES = BN * BK / 2;     // 32 KB
constexpr int SFA_BYTES = BM * BK / 16;  // 2 KB
constexpr int SFB_BYTES = BN * BK / 16;  // 4 KB
constexpr int SF_LAG = STAGES - 1;       // scale stages in flight before the first shuffle
constexpr int TMEM_COLS = 512;
constexpr uint32_t COL_SFA = 256;
constexpr uint32_t COL_SFB = 272;

struct alignas(1024) Smem {
  uint8_t a[STAGES][A_BYTES];
  uint8_t b[STAGES][B_BYTES];
  alignas(128) uint8_t sfa[STAGES][SFA_BYTES];
  alignas(128) uint8_t sfb[STAGES][SFB_BYTES];
  uint64_t full[STAGES];     // A/B landed (1 arrival + tx bytes)
  uint64_t sf_full[STAGES];  // scale factors landed and shuffled (1 arrival from the SF warp)
  uint64_t empty[STAGES];    // 1 arrival (MMA commit)
  uint64_t sf_raw[STAGES];   // SF TMA landed (1 arrival + tx)
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint64_t mma_done;
  UnitQueue<Q> queue;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;

__device__ __forceinline__ Smem& smem_ref(uint8_t* raw) {
  uintptr_t p = reinterpret_cast<uintptr_t>(raw);
  p = (p + 1023) & ~static_cast<uintptr_t>(1023);
  return *reinterpret_cast<Smem*>(p);
}

// In-place shuffle of one 128-row block of scale bytes (row r at r*16, 16 bytes = 4 MMA steps x 4
// scales) into 4 consecutive 512-byte blocks, one per MMA step k, where the 16 bytes at l*16 hold
// the 4 scales of rows l, l+32, l+64, l+96 for that step.  One warp; all reads precede all writes.
__device__ __forceinline__ void shuffle_sf_block(uint8_t* blk) {
  const int l = lane_idx();
  uint4 w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) w[q] = *reinterpret_cast<const uint4*>(blk + (q * 32 + l) * 16);
  __syncwarp();
  uint4 o0 = make_uint4(w[0].x, w[1].x, w[2].x, w[3].x);
  uint4 o1 = make_uint4(w[0].y, w[1].y, w[2].y, w[3].y);
  uint4 o2 = make_uint4(w[0].z, w[1].z, w[2].z, w[3].z);
  uint4 o3 = make_uint4(w[0].w, w[1].w, w[2].w, w[3].w);
  *reinterpret_cast<uint4*>(blk + 0 * 512 + l * 16) = o0;
  *reinterpret_cast<uint4*>(blk + 1 * 512 + l * 16) = o1;
  *reinterpret_cast<uint4*>(blk + 2 * 512 + l * 16) = o2;
  *reinterpret_cast<uint4*>(blk + 3 * 512 + l * 16) = o3;
}

__global__ void __launch_bounds__(THREADS, 1) bsg_nvfp4_grouped_kernel(const __grid_constant__ Nvfp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = smem_ref(smem_raw);
  const int warp = warp_idx();
  const int lane = lane_idx();
  const int KS = p.K / BK;
  const int n_tiles = (p.N + BN - 1) / BN;
  WaitCtx wctx{p.timeout_ns, &s.abort, p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.sf_full[i], 1);
      mbar_init(&s.empty[i], 1);
      mbar_init(&s.sf_raw[i], 1);
    }
    mbar_init(&s.mma_done, 1);
    mbar_init(&s.tmem_full, 1);
    mbar_init(&s.tmem_empty, EPI_WARPS);
    for (int i = 0; i < Q; ++i) {
      mbar_init(&s.queue.full[i], 1);
      mbar_init(&s.queue.empty[i], EPI_WARPS + 3);
    }
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == WARP_SF && lane == 0) {
    tma_prefetch_desc(&p.tmSFA);
    tma_prefetch_desc(&p.tmSFB);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;

  if (warp == WARP_SCHED) {
    run_scheduler<Q, BN, false>(s.queue, p.m_indices, p.M, p.G, n_tiles, p.n_group, wctx, p.debug_mode);
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
          mbar_arrive_expect_tx(&s.full[pos.stage], A_BYTES + B_BYTES);
          tma_load_2d(s.a[pos.stage], &p.tmA, &s.full[pos.stage], kb * (BK / 2), u.row0);
          tma_load_3d(s.b[pos.stage], &p.tmB, &s.full[pos.stage], kb * (BK / 2), u.n0, u.g);
        }
        __syncwarp();
        ++issued;
        pos.advance();
      }
    }
    if (ok) {
      for (int i = 0; i < STAGES; ++i) {
        if (!mbar_wait(&s.empty[pos.stage], pos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status, kSiteDrain,
                       pos.stage))
          break;
        pos.advance();
      }
    } else {
      drain_inflight_loads<STAGES>(s.full, pos, issued, wctx);
    }
  } else if (warp == WARP_SF) {
    // Issue the scale loads of step i, then shuffle the oldest step once SF_LAG are outstanding (the
    // TMA latency of the later steps overlaps).  Steps run over all units of the CTA in order.
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;     // next step to issue
    RingPos<STAGES> old;     // oldest issued, not yet shuffled
    long long issued = 0;
    int pending = 0;
    bool ok = true;
    auto process_oldest = [&]() -> bool {
      if (!mbar_wait(&s.sf_raw[old.stage], old.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSfRaw,
                     old.stage))
        return false;
      shuffle_sf_block(s.sfa[old.stage]);
      shuffle_sf_block(s.sfb[old.stage]);
      shuffle_sf_block(s.sfb[old.stage] + 2048);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.sf_full[old.stage]);
      old.advance();
      --pending;
      return true;
    };
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
          mbar_arrive_expect_tx(&s.sf_raw[pos.stage], SFA_BYTES + SFB_BYTES);
          tma_load_2d(s.sfa[pos.stage], &p.tmSFA, &s.sf_raw[pos.stage], kb * (BK / 16), u.row0);
          tma_load_3d(s.sfb[pos.stage], &p.tmSFB, &s.sf_raw[pos.stage], kb * (BK / 16), u.n0, u.g);
        }
        __syncwarp();
        ++issued;
        pos.advance();
        if (++pending >= SF_LAG && !process_oldest()) {
          ok = false;
          break;
        }
      }
    }
    while (ok && pending > 0) {
      if (!process_oldest()) ok = false;
    }
    if (!ok) drain_inflight_loads<STAGES>(s.sf_raw, pos, issued, wctx);
  } else if (warp == WARP_MMA) {
    constexpr uint32_t IDESC = idesc_mxf4nvf4(BM, BN);
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    uint32_t acc_phase = 0;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      if (!mbar_wait(&s.tmem_empty, acc_phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status, kSiteTmemEmpty, 0))
        break;
      tc_fence_after();
      for (int kb = 0; kb < KS; ++kb) {
        if (!mbar_wait(&s.full[pos.stage], pos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSmemFull,
                       pos.stage) ||
            !mbar_wait(&s.sf_full[pos.stage], pos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSmemFull,
                       pos.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = sdesc_k_sw128(smem_u32(s.a[pos.stage]));
          const uint64_t db = sdesc_k_sw128(smem_u32(s.b[pos.stage]));
          const uint32_t sfa_s = smem_u32(s.sfa[pos.stage]);
          const uint32_t sfb_s = smem_u32(s.sfb[pos.stage]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            tc_cp_32x128b_warpx4(tmem_base + COL_SFA + 4 * k, sdesc_sf(sfa_s + k * 512));
            tc_cp_32x128b_warpx4(tmem_base + COL_SFB + 8 * k, sdesc_sf(sfb_s + k * 512));
            tc_cp_32x128b_warpx4(tmem_base + COL_SFB + 8 * k + 4, sdesc_sf(sfb_s + 2048 + k * 512));
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mma_mxf4nvf4(tmem_base, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k), IDESC,
                         tmem_base + COL_SFA + 4 * k, tmem_base + COL_SFB + 8 * k, (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&s.empty[pos.stage]);
          if (kb == KS - 1) tc_commit(&s.tmem_full);
        }
        __syncwarp();
        pos.advance();
      }
      acc_phase ^= 1u;
    }
    if (lane == 0) tc_commit(&s.mma_done);
    __syncwarp();
    mbar_wait(&s.mma_done, 0, wctx.timeout_ns, nullptr, nullptr, kSiteDrain, 0);
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
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 128; c += 16) {
        uint32_t t[16];
        tmem_ld_x16(taddr + c, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[c + i] = t[i];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tmem_empty);
      acc_phase ^= 1u;
      const int row = u.row0 + r;
      const int col0 = u.n0 + half * 128;
      if (row >= u.row_lo && row < u.row_hi && col0 < p.N) {
        const int ncols = min(128, p.N - col0);
        __nv_bfloat16* dst = p.C + static_cast<size_t>(row) * p.N + col0;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          if (c < ncols) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[c + 0]) * alpha, __uint_as_float(v[c + 1]) * alpha);
            o.y = pack_bf16x2(__uint_as_float(v[c + 2]) * alpha, __uint_as_float(v[c + 3]) * alpha);
            o.z = pack_bf16x2(__uint_as_float(v[c + 4]) * alpha, __uint_as_float(v[c + 5]) * alpha);
            o.w = pack_bf16x2(__uint_as_float(v[c + 6]) * alpha, __uint_as_float(v[c + 7]) * alpha);
            *reinterpret_cast<uint4*>(dst + c) = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_MMA) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace nvfp4
}  // namespace bsg
