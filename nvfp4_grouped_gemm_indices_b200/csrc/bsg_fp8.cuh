// bsg_fp8.cuh -- FP8 (E4M3) grouped GEMM with FP32 per-128 block scales, BF16 out, sm_100a.
//
// Operation: the FP8 page ("[flashinfer] FlashInfer FP8 GEMM 최적화: 윈도우 세그먼트 KG1 프로그램으로
// GPU 성능 극대화", introduction and section 1):
//   C[m, n] = bf16( sum_kb a_scale[m, kb] * b_scale[g, n/128, kb] * (A[m, kb-block] . B[g, n, kb-block]) )
//
// Design (persistent, warp-specialised, one CTA per SM):
//   warps 0..7  epilogue: warp w owns TMEM lanes 32*(w%4).. (tile rows) and columns 128*(w/4)..;
//               per K block it reads the fresh FP32 partial from TMEM, multiplies by
//               a_scale[row, kb] * b_scale[g, col/128, kb] and accumulates in registers; after the
//               last K block it rounds to BF16 and stores the rows of the segment only.
//   warp 8      TMA producer: A box [128 rows x 128 B] of the window, B box [BN rows x 128 B] of
//               expert g, into an N-stage shared-memory ring (full/empty mbarriers).
//   warp 9      TMEM allocator + single-thread tcgen05.mma issuer: 4 x (128 x BN x 32) kind::f8f6f4
//               MMAs per 128-K block into a fresh accumulator; two accumulators ping-pong so the
//               tensor core works on block kb+1 while the epilogue promotes block kb.
//   warp 10     scheduler (bsg_sched.cuh): window segmentation and unit hand-out.
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
  CUtensorMap tmB;  // uint8 [G, N, K]: dims {K, N, G}, box {128, BN, 1}, 128B swizzle
  const float* a_scale;
  const float* b_scale;
  const int* m_indices;
  __nv_bfloat16* C;
  int M, N, K, G;
  uint64_t timeout_ns;
  DeviceStatus* status;
  int debug_mode;
};

namespace fp8 {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;                 // one scale block
constexpr int STAGES = 4;
constexpr int ACC = 2;                  // TMEM accumulators (ping-pong per K block)
constexpr int Q = 4;                    // unit queue depth
constexpr int EPI_WARPS = 8;
constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_SCHED = 10;
constexpr int NUM_WARPS = 11;
constexpr int THREADS = NUM_WARPS * 32;
constexpr int A_BYTES = BM * BK;        // 16 KB
constexpr int B_BYTES = BN * BK;        // 32 KB
constexpr int TMEM_COLS = 512;

struct alignas(1024) Smem {
  uint8_t a[STAGES][A_BYTES];
  uint8_t b[STAGES][B_BYTES];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[ACC];
  uint64_t tmem_empty[ACC];
  uint64_t mma_done;
  UnitQueue<Q> queue;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;  // + alignment slack

__device__ __forceinline__ Smem& smem_ref(uint8_t* raw) {
  uintptr_t p = reinterpret_cast<uintptr_t>(raw);
  p = (p + 1023) & ~static_cast<uintptr_t>(1023);
  return *reinterpret_cast<Smem*>(p);
}

__global__ void __launch_bounds__(THREADS, 1) kernel(const __grid_constant__ Fp8Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = smem_ref(smem_raw);
  const int warp = warp_idx();
  const int lane = lane_idx();
  const int KB = p.K / BK;
  const int n_tiles = (p.N + BN - 1) / BN;
  WaitCtx wctx{p.timeout_ns, &s.abort, p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < ACC; ++i) {
      mbar_init(&s.tmem_full[i], 1);
      mbar_init(&s.tmem_empty[i], EPI_WARPS);
    }
    for (int i = 0; i < Q; ++i) {
      mbar_init(&s.queue.full[i], 1);
      mbar_init(&s.queue.empty[i], EPI_WARPS + 2);
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
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;

  if (warp == WARP_SCHED) {
    run_scheduler<Q, BN>(s.queue, p.m_indices, p.M, p.G, n_tiles, wctx, p.debug_mode);
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
          mbar_arrive_expect_tx(&s.full[pos.stage], A_BYTES + B_BYTES);
          tma_load_2d(s.a[pos.stage], &p.tmA, &s.full[pos.stage], kb * BK, u.row0);
          tma_load_3d(s.b[pos.stage], &p.tmB, &s.full[pos.stage], kb * BK, u.n0, u.g);
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
      drain_inflight_loads<STAGES>(s.full, pos, issued, wctx);
    }
  } else if (warp == WARP_MMA) {
    constexpr uint32_t IDESC = idesc_f8f6f4_e4m3(BM, BN);
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    RingPos<ACC> accp;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.tmem_empty[accp.stage], accp.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteTmemEmpty, accp.stage) ||
            !mbar_wait(&s.full[pos.stage], pos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteSmemFull,
                       pos.stage)) {
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
            mma_f8f6f4(d_tmem, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k), IDESC,
                       k > 0 ? 1u : 0u);
          }
          tc_commit(&s.empty[pos.stage]);
          tc_commit(&s.tmem_full[accp.stage]);
        }
        __syncwarp();
        pos.advance();
        accp.advance();
      }
    }
    // every MMA this thread issued has completed before TMEM may be released
    if (lane == 0) tc_commit(&s.mma_done);
    __syncwarp();
    mbar_wait(&s.mma_done, 0, wctx.timeout_ns, nullptr, nullptr, kSiteDrain, 0);
  } else {
    // ------------------------------------------------------------------ epilogue warps 0..7
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int r = quarter * 32 + lane;                  // tile row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int NB = (p.N + 127) / 128;
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<ACC> accp;
    while (true) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      const int row = u.row0 + r;
      const bool row_ok = row < p.M;
      const int col0 = u.n0 + half * 128;
      const int nb = col0 / 128;
      const float* sa_ptr = p.a_scale + static_cast<size_t>(row_ok ? row : 0) * KB;
      const float* sb_ptr = p.b_scale + (static_cast<size_t>(u.g) * NB + (nb < NB ? nb : NB - 1)) * KB;
      float accum[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) accum[i] = 0.f;
      float sa_next = row_ok ? __ldg(sa_ptr) : 0.f;
      float sb_next = __ldg(sb_ptr);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const float scale = sa_next * sb_next;
        if (kb + 1 < KB) {
          sa_next = row_ok ? __ldg(sa_ptr + kb + 1) : 0.f;
          sb_next = __ldg(sb_ptr + kb + 1);
        }
        if (!mbar_wait(&s.tmem_full[accp.stage], accp.phase, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteTmemFull, accp.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + static_cast<uint32_t>(accp.stage * BN + half * 128);
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
          uint32_t v0[16], v1[16];
          tmem_ld_x16(taddr + c, v0);
          tmem_ld_x16(taddr + c + 16, v1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            accum[c + i] = fmaf(__uint_as_float(v0[i]), scale, accum[c + i]);
            accum[c + 16 + i] = fmaf(__uint_as_float(v1[i]), scale, accum[c + 16 + i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tmem_empty[accp.stage]);
        accp.advance();
      }
      if (!ok) break;
      // masked BF16 store of this thread's row: only rows of the segment, only columns < N
      if (row >= u.row_lo && row < u.row_hi && col0 < p.N) {
        const int ncols = min(128, p.N - col0);
        __nv_bfloat16* dst = p.C + static_cast<size_t>(row) * p.N + col0;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
          if (c < ncols) {
            uint4 v;
            v.x = pack_bf16x2(accum[c + 0], accum[c + 1]);
            v.y = pack_bf16x2(accum[c + 2], accum[c + 3]);
            v.z = pack_bf16x2(accum[c + 4], accum[c + 5]);
            v.w = pack_bf16x2(accum[c + 6], accum[c + 7]);
            *reinterpret_cast<uint4*>(dst + c) = v;
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

}  // namespace fp8
}  // namespace bsg
