// bsg_fp8_swap.cuh -- FP8 grouped GEMM for experts with few rows (decode): the operands of the MMA
// are swapped so that the token count, not a 128-row window, sets the MMA shape.
//
// Same operation and inputs as bsg_fp8.cuh (the FP8 page, "[flashinfer] FlashInfer FP8 GEMM 최적화:
// 윈도우 세그먼트 KG1 프로그램으로 GPU 성능 극대화", introduction and section 1):
//   C[m, n] = bf16( sum_kb a_scale[m, kb] * b_scale[g, n/128, kb] * (A[m, kb-block] . B[g, n, kb-block]) )
// computed as its transpose, C^T[n, m] = B[g] . A^T: the tcgen05 MMA's 128-row operand is 128 rows
// of B[g] (output columns), its N operand is the segment's tokens, N = 16 * ceil(tokens / 16).  With
// 1-3 tokens per expert (the skewed decode routing) the MMAs and the promotion shrink ~8x against a
// 128 x 256 row tile, and the kernel is left streaming B from HBM.  The page "[onnxruntime] ONNX
// Runtime: Blackwell (SM120+)에서 NVFP4 QMoE를 위한 네이티브 FP4xFP4 Prefill 최적화", section 1,
// keeps decode / small-M shapes on their own latency-oriented path and picks the prefill GEMM by
// token count; here that path is this operand-swapped tensor-core GEMM on the same block-scaled
// operands (its dequantising A16 runner is a fallback and is not built), picked by the chooser.
//
// Template NH: B rows per unit = 128 * NH (NH MMAs per K step, one per 128-row half), token tile
// TM = 128 / NH.  Units come from the window scheduler (bsg_sched.cuh) with segments cut into chunks
// of at most TM tokens: (token chunk [lo, hi) of expert g, 128 * NH output columns at n0).
// Roles (20 warps, one CTA per SM, persistent):
//   warp 0      TMA: B[g] rows n0 .. n0 + 128 NH (one box) and ceil(tokens / 16) boxes of 16 A rows
//               starting at row lo, per 128-K block, into a STAGES-deep ring.
//   warp 1      TMEM allocator + single-thread MMA issuer: per K block 4 K steps x NH MMAs of
//               128 x N x 32 (kind::f8f6f4) into a fresh accumulator; four 128-column accumulators
//               rotate between the MMAs and the promotion.
//   warp 2      scheduler.   warp 3  scale producer (a_scale of the chunk's tokens, b_scale of the
//               NH 128-column blocks, by cp.async into a scale ring).
//   warps 4..19 promotion + store: warp w reads TMEM lane quarter w % 4 (32 output columns) and 32
//               token columns; per K block acc[t] += partial[t] * a_scale[token t, kb] * b_scale[kb];
//               warps whose token columns are all past the chunk only keep the barriers moving.
//               The store writes C[token, n] for tokens of the chunk and n < N.
#pragma once

#include <cuda_bf16.h>

#include "bsg_ptx.cuh"
#include "bsg_sched.cuh"
#include "bsg_fp8.cuh"

namespace bsg {
namespace fp8s {

constexpr int BK = 128;                 // one scale block
constexpr int A_BOX = 16;               // token rows per TMA box of A
constexpr int SC_STAGES = 12;
constexpr int Q = 4;
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_SCHED = 2, WARP_SCALE = 3, WARP_EPI0 = 4;
constexpr int EPI_WARPS = 16;
constexpr int NUM_WARPS = WARP_EPI0 + EPI_WARPS;
constexpr int THREADS = NUM_WARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 128;           // NH halves x TM token columns
constexpr int ACC = TMEM_COLS / ACC_COLS;
constexpr int EPI_COLS = 32;            // token columns per epilogue warp

template <int NH>
struct Cfg {
  static constexpr int BNR = 128 * NH;          // B rows (output columns) per unit
  static constexpr int TM = 128 / NH;           // tokens per unit at most
  static constexpr int A_BYTES = TM * BK;       // 16 KB / 8 KB
  static constexpr int B_BYTES = BNR * BK;      // 16 KB / 32 KB
  static constexpr int STAGES = NH == 1 ? 6 : 5;
};

struct ScaleSlot {
  float a[128];        // a_scale[lo + t, kb], zero past the chunk (up to the next multiple of 32)
  float b[2];          // b_scale[g, n0 / 128 + h, kb]
  float pad[2];
};

template <int NH>
struct alignas(1024) Smem {
  uint8_t a[Cfg<NH>::STAGES][Cfg<NH>::A_BYTES];
  uint8_t b[Cfg<NH>::STAGES][Cfg<NH>::B_BYTES];
  ScaleSlot sc[SC_STAGES];
  uint64_t full[Cfg<NH>::STAGES];
  uint64_t empty[Cfg<NH>::STAGES];
  uint64_t sc_full[SC_STAGES];
  uint64_t sc_empty[SC_STAGES];
  uint64_t tmem_full[ACC];
  uint64_t tmem_empty[ACC];
  uint64_t mma_done;
  UnitQueue<Q> queue;
  uint32_t tmem_base;
  int abort;
};

template <int NH>
constexpr size_t smem_bytes() {
  return sizeof(Smem<NH>) + 1024;
}

template <int NH>
__device__ __forceinline__ Smem<NH>& smem_ref(uint8_t* raw) {
  uintptr_t p = reinterpret_cast<uintptr_t>(raw);
  p = (p + 1023) & ~static_cast<uintptr_t>(1023);
  return *reinterpret_cast<Smem<NH>*>(p);
}

template <int NH>
__device__ __forceinline__ void fp8_swap_body(const Fp8Params& p) {
  using C = Cfg<NH>;
  constexpr int STAGES = C::STAGES;
  constexpr int TM = C::TM;
  extern __shared__ uint8_t smem_raw[];
  Smem<NH>& s = smem_ref<NH>(smem_raw);
  const int warp = warp_idx();
  const int lane = lane_idx();
  const int KB = p.K / BK;
  const int n_tiles = (p.N + C::BNR - 1) / C::BNR;
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
    for (int i = 0; i < ACC; ++i) {
      mbar_init(&s.tmem_full[i], 1);
      mbar_init(&s.tmem_empty[i], EPI_WARPS);
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
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;
  // Small launches run as programmatic dependents of the previous kernel on the stream: the set-up
  // above overlapped it; wait for it to complete (its writes visible) before touching global memory,
  // then let the next kernel start its own set-up.  Without that launch attribute both are no-ops.
  grid_dependency_wait();
  grid_dependents_launch();

  if (warp == WARP_SCHED) {
    run_scheduler<Q, C::BNR, false, TM>(s.queue, p.m_indices, p.M, p.G, n_tiles, p.n_group, wctx, p.debug_mode);
  } else if (warp == WARP_SCALE) {
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
      const int cnt = u.row_hi - u.row_lo;        // 1 .. TM
      const int rounds = (cnt + 31) / 32;
      const int nb0 = u.n0 / 128;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.sc_empty[spos.stage], spos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteSmemEmpty, 16 + spos.stage)) {
          ok = false;
          break;
        }
        ScaleSlot& slot = s.sc[spos.stage];
        for (int i = 0; i < rounds; ++i) {
          const int t = i * 32 + lane;
          const bool in = t < cnt;
          fp8::cp_async_4(&slot.a[t], p.a_scale + static_cast<size_t>(in ? u.row_lo + t : 0) * KB + kb, in ? 4u : 0u);
        }
        if (lane < NH) {
          const bool in = nb0 + lane < NB;
          fp8::cp_async_4(&slot.b[lane],
                          p.b_scale + (static_cast<size_t>(u.g) * NB + (in ? nb0 + lane : 0)) * KB + kb,
                          in ? 4u : 0u);
        }
        fp8::cp_async_arrive(&s.sc_full[spos.stage]);
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
      const int nbox = (u.row_hi - u.row_lo + A_BOX - 1) / A_BOX;   // 1 .. TM / 16
      const uint32_t tx = static_cast<uint32_t>(C::B_BYTES + nbox * A_BOX * BK);
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.empty[pos.stage], pos.phase ^ 1u, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteSmemEmpty, pos.stage)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&s.full[pos.stage], tx);
          tma_load_3d(s.b[pos.stage], &p.tmB, &s.full[pos.stage], kb * BK, u.n0, u.g);
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(s.a[pos.stage] + i * A_BOX * BK, &p.tmA, &s.full[pos.stage], kb * BK, u.row_lo + i * A_BOX);
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
  } else if (warp == WARP_MMA) {
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<STAGES> pos;
    RingPos<ACC> accp;
    bool ok = true;
    while (ok) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      const int nmma = A_BOX * ((u.row_hi - u.row_lo + A_BOX - 1) / A_BOX);   // MMA N: 16 .. TM
      const uint32_t idesc = idesc_f8f6f4_e4m3(128, nmma);
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
          const uint64_t dx = sdesc_k_sw128(smem_u32(s.a[pos.stage]));     // tokens: the MMA's N operand
          const uint32_t d0 = tmem_base + static_cast<uint32_t>(accp.stage * ACC_COLS);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              // B rows 128h .. 128h + 127 of the stage: the MMA's 128-row operand
              const uint64_t dw = sdesc_k_sw128(smem_u32(s.b[pos.stage] + h * 128 * BK));
              mma_f8f6f4(d0 + static_cast<uint32_t>(h * TM), dw + static_cast<uint64_t>(2 * k),
                         dx + static_cast<uint64_t>(2 * k), idesc, k > 0 ? 1u : 0u);
            }
          }
          tc_commit(&s.empty[pos.stage]);
          tc_commit(&s.tmem_full[accp.stage]);
        }
        __syncwarp();
        pos.advance();
        accp.advance();
      }
    }
    if (lane == 0) tc_commit(&s.mma_done);
    __syncwarp();
    mbar_wait(&s.mma_done, 0, wctx.timeout_ns, nullptr, nullptr, kSiteDrain, 0);
  } else if (warp >= WARP_EPI0) {
    const int quarter = warp & 3;                   // TMEM lane quarter: output columns 32q .. 32q + 31
    const int cg = (warp - WARP_EPI0) >> 2;         // 0 .. 3
    const int h = NH == 1 ? 0 : (cg >> 1);          // which 128-row half of the unit's B rows
    const int t0 = NH == 1 ? cg * EPI_COLS : (cg & 1) * EPI_COLS;   // first token column of this warp
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int qslot = 0;
    uint32_t qphase = 0;
    RingPos<ACC> accp;
    RingPos<SC_STAGES> spos;
    while (true) {
      Unit u;
      if (!queue_pop(s.queue, qslot, qphase, u, wctx) || !u.valid) break;
      const int cnt = u.row_hi - u.row_lo;
      const int ncols = min(max(cnt - t0, 0), EPI_COLS);   // token columns of this warp in the chunk
      float2 acc[EPI_COLS / 2];
#pragma unroll
      for (int i = 0; i < EPI_COLS / 2; ++i) acc[i] = make_float2(0.f, 0.f);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&s.sc_full[spos.stage], spos.phase, wctx.timeout_ns, wctx.abort, wctx.status, kSiteTmemFull,
                       16 + spos.stage)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&s.tmem_full[accp.stage], accp.phase, wctx.timeout_ns, wctx.abort, wctx.status,
                       kSiteTmemFull, accp.stage)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const ScaleSlot& sl = s.sc[spos.stage];
        const float bs = sl.b[h];
        const uint32_t taddr =
            tmem_base + lane_addr + static_cast<uint32_t>(accp.stage * ACC_COLS + h * TM + t0);
#pragma unroll
        for (int c = 0; c < EPI_COLS; c += 16) {
          if (c < ncols) {
            uint32_t v[16];
            tmem_ld_x16(taddr + c, v);
            float2 sv[8];   // a_scale * b_scale of the chunk's 16 tokens, read while the TMEM load runs
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 a4 = *reinterpret_cast<const float4*>(sl.a + t0 + c + 4 * j);
              sv[2 * j] = make_float2(a4.x * bs, a4.y * bs);
              sv[2 * j + 1] = make_float2(a4.z * bs, a4.w * bs);
            }
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              acc[c / 2 + i] = __ffma2_rn(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])),
                                          sv[i], acc[c / 2 + i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&s.sc_empty[spos.stage]);
          mbar_arrive(&s.tmem_empty[accp.stage]);
        }
        spos.advance();
        accp.advance();
      }
      if (!ok) break;
      // C[token, n]: this thread's output column n, the warp's tokens of the chunk
      const int n = u.n0 + h * 128 + quarter * 32 + lane;
      if (n < p.N && ncols > 0) {
        __nv_bfloat16* dst = p.C + static_cast<size_t>(u.row_lo + t0) * p.N + n;
#pragma unroll
        for (int j = 0; j < EPI_COLS; ++j) {
          if (j < ncols) {
            const float v = (j & 1) ? acc[j / 2].y : acc[j / 2].x;
            dst[static_cast<size_t>(j) * p.N] = __float2bfloat16_rn(v);
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

__global__ void __launch_bounds__(THREADS, 1) bsg_fp8_swap_kernel(const __grid_constant__ Fp8Params p) {
  fp8_swap_body<1>(p);
}

__global__ void __launch_bounds__(THREADS, 1) bsg_fp8_swap_n256_kernel(const __grid_constant__ Fp8Params p) {
  fp8_swap_body<2>(p);
}

}  // namespace fp8s
}  // namespace bsg
