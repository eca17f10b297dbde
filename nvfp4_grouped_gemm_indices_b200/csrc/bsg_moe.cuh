// bsg_moe.cuh -- the MoE expand permutation: the (token, choice) routing entries laid out expert by
// expert, so that each expert's rows form one contiguous run of the grouped GEMM's A (the expanded
// input rows of the page "[onnxruntime] ONNX Runtime: Blackwell (SM120+)에서 NVFP4 QMoE를 위한 네이티브
// FP4xFP4 Prefill 최적화", section 1, which quantises those rows on the way).
//
// Operation: a stable counting sort of the n = T * top_k entries i = t * top_k + k by their expert
// g = expert_ids[i] in [0, G):
//     src_rows[p] = t, m_indices[p] = g, dst_rows[i] = p   (p runs through g's run in increasing i)
//     expert_offsets[g] = first position of g's run; expert_offsets[G] = entries placed
// entries with an expert outside [0, G) are dropped (dst_rows = -1) and the positions past the last
// placed entry hold -1 in src_rows and m_indices (rows the GEMM skips and the quantiser leaves alone).
//
// Design: the entries are cut into `tiles` consecutive tiles of `tile` entries, one warp per tile,
// WARPS warps per CTA; the scratch holds one row of G counters per tile (tiles x G int32).
//   1. count:   each warp counts its tile's entries per expert in its own shared-memory row (one
//               32-entry group at a time: __match_any_sync groups the lanes with equal experts and the
//               group's first lane adds the group's size), then writes the row to the scratch.
//   2. scan:    one CTA turns the counts into starting positions: per expert the sum over tiles, an
//               exclusive scan over experts (expert_offsets), then per expert the running sum down the
//               tiles (the scratch row of tile w now holds where w's entries of each expert begin);
//               the tiles are cut into segments so that all its threads walk columns of counters.
//   3. scatter: each warp walks its tile again in order with its row of starting positions in
//               shared memory; an entry's position is its group's base plus its rank among the
//               group's lanes, and the group's first lane advances the base -- so entries of one
//               expert keep their token order (stable) inside a tile, across tiles by the scan.
//               The kernel also fills the unused tail positions with -1.
// Small problems (n <= FUSED_MAX_N entries, G <= FUSED_MAX_G experts) take the same three steps in one
// launch of one 1024-thread CTA (bsg_moe_fused_kernel): the 32 tiles' counter rows live in shared
// memory, so there is no scratch in global memory and no dependent launch; each lane loads BATCH
// entries ahead so the loads of a tile overlap.
// The counting is integer work bound by the latency of its dependent steps, not by a roofline; all
// memory traffic is coalesced except the scattered 4-byte output writes.
#pragma once

#include <cstdint>

namespace bsg {
namespace moe {

constexpr int WARPS = 4;                 // warps (tiles) per CTA of the count and scatter kernels
constexpr int THREADS = WARPS * 32;
constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_BATCH = 16;           // counters each scan thread loads ahead
constexpr int MAX_TILES = 512;           // at most MAX_TILES x G counters for the one-CTA scan
constexpr int MIN_TILE = 256;            // entries per tile when the scratch allows it
constexpr int FUSED_THREADS = 1024;      // the single-CTA path: 32 warps, one tile each
constexpr int FUSED_WARPS = FUSED_THREADS / 32;
constexpr long long FUSED_MAX_N = 4096;      // measured crossover (graph replay): 11.7 vs 12.5 us at 4096, 16.2 vs 13.4 at 8192
constexpr int FUSED_MAX_G = FUSED_THREADS;   // one thread per expert in the scan
constexpr int BATCH = 16;                // 32-entry groups each lane of the single-CTA path loads ahead

struct Params {
  const int32_t* expert_ids;  // [n]
  int32_t* src_rows;          // [n]
  int32_t* m_indices;         // [n]
  int32_t* dst_rows;          // [n]
  int32_t* expert_offsets;    // [G + 1]
  int32_t* scratch;           // [tiles, G]
  long long n;
  int top_k, G;
  int tile, tiles;
};

// Programmatic dependent launch: the scan and scatter kernels are launched while their predecessor
// still runs, so their launch latency overlaps it; `dependency_wait` blocks until the predecessor
// grid has completed and its memory writes are visible, `allow_dependents` lets the next grid start
// its launch early.
__device__ __forceinline__ void dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ int32_t expert_at(const Params& p, long long i) {
  const int32_t g = __ldg(p.expert_ids + i);
  return (g >= 0 && g < p.G) ? g : -1;
}

// Per-tile expert counts; dynamic shared memory: WARPS x G int32.
__global__ void __launch_bounds__(THREADS) bsg_moe_count_kernel(const __grid_constant__ Params p) {
  extern __shared__ int32_t moe_smem[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int w = blockIdx.x * WARPS + wib;
  int32_t* row = moe_smem + static_cast<size_t>(wib) * p.G;
  allow_dependents();
  if (w >= p.tiles) return;                              // warp-uniform
  for (int g = lane; g < p.G; g += 32) row[g] = 0;
  __syncwarp();
  const int i0 = w * p.tile;
  const int i1 = static_cast<int>(min(p.n, static_cast<long long>(i0) + p.tile));
  for (int base = i0; base < i1; base += 32 * BATCH) {
    int32_t g[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {            // the batch's loads are all in flight before the first use
      const int i = base + 32 * j + lane;
      g[j] = i < i1 ? expert_at(p, i) : -1;
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const unsigned peers = __match_any_sync(0xffffffffu, g[j]);
      if (g[j] >= 0 && lane == __ffs(peers) - 1) row[g[j]] += __popc(peers);
      __syncwarp();
    }
  }
  int32_t* out = p.scratch + static_cast<size_t>(w) * p.G;
  for (int g = lane; g < p.G; g += 32) out[g] = row[g];
}

// One CTA: expert_offsets (exclusive scan over experts of the per-expert totals) and, in place of
// each tile's counts, the position where that tile's entries of each expert begin.  With G <=
// SCAN_THREADS the tiles are cut into S = SCAN_THREADS / G segments so that every thread walks one
// (segment, expert) column; with more experts each thread takes several experts (S = 1).  Dynamic
// shared memory: (S * G + G) int32 -- the segment sums, then the experts' starting positions.
__global__ void __launch_bounds__(SCAN_THREADS) bsg_moe_scan_kernel(const __grid_constant__ Params p) {
  extern __shared__ int32_t moe_smem[];
  __shared__ int32_t part[SCAN_THREADS];
  const int tid = threadIdx.x;
  const int G = p.G;
  const int S = G <= SCAN_THREADS ? SCAN_THREADS / G : 1;
  const int seg = (p.tiles + S - 1) / S;
  allow_dependents();
  dependency_wait();                                     // the count kernel's rows are complete
  int32_t* seg_sum = moe_smem;                          // [S][G]
  int32_t* start = moe_smem + S * G;                     // [G]
  // 1. each (segment, expert) column's sum
  for (int item = tid; item < S * G; item += SCAN_THREADS) {
    const int g = item % G;
    const int w0 = (item / G) * seg;
    const int w1 = min(p.tiles, w0 + seg);
    int32_t sum = 0;
    int w = w0;
    for (; w + SCAN_BATCH <= w1; w += SCAN_BATCH) {      // SCAN_BATCH independent loads in flight
      int32_t v[SCAN_BATCH];
#pragma unroll
      for (int j = 0; j < SCAN_BATCH; ++j) v[j] = p.scratch[static_cast<size_t>(w + j) * G + g];
#pragma unroll
      for (int j = 0; j < SCAN_BATCH; ++j) sum += v[j];
    }
    for (; w < w1; ++w) sum += p.scratch[static_cast<size_t>(w) * G + g];
    seg_sum[item] = sum;
  }
  __syncthreads();
  for (int g = tid; g < G; g += SCAN_THREADS) {
    int32_t t = 0;
    for (int q = 0; q < S; ++q) t += seg_sum[q * G + g];
    start[g] = t;
  }
  __syncthreads();
  // 2. exclusive scan of start[0, G): thread tid owns the consecutive experts [tid * per, +per)
  const int per = (G + SCAN_THREADS - 1) / SCAN_THREADS;
  const int g0 = tid * per;
  int32_t local = 0;
  for (int j = 0; j < per && g0 + j < G; ++j) local += start[g0 + j];
  part[tid] = local;
  __syncthreads();
  for (int off = 1; off < SCAN_THREADS; off <<= 1) {     // inclusive Hillis-Steele scan of part[]
    const int32_t v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int32_t run = part[tid] - local;                       // exclusive prefix of this thread's experts
  for (int j = 0; j < per && g0 + j < G; ++j) {
    const int32_t c = start[g0 + j];
    start[g0 + j] = run;
    p.expert_offsets[g0 + j] = run;
    run += c;
  }
  if (tid == SCAN_THREADS - 1) p.expert_offsets[G] = part[SCAN_THREADS - 1];
  __syncthreads();
  // 3. the running sum down each column, from the expert's start plus the earlier segments' sums
  for (int item = tid; item < S * G; item += SCAN_THREADS) {
    const int g = item % G;
    const int q = item / G;
    const int w0 = q * seg;
    const int w1 = min(p.tiles, w0 + seg);
    int32_t r = start[g];
    for (int e = 0; e < q; ++e) r += seg_sum[e * G + g];
    int w = w0;
    for (; w + SCAN_BATCH <= w1; w += SCAN_BATCH) {
      int32_t v[SCAN_BATCH];
#pragma unroll
      for (int j = 0; j < SCAN_BATCH; ++j) v[j] = p.scratch[static_cast<size_t>(w + j) * G + g];
#pragma unroll
      for (int j = 0; j < SCAN_BATCH; ++j) {
        p.scratch[static_cast<size_t>(w + j) * G + g] = r;
        r += v[j];
      }
    }
    for (; w < w1; ++w) {
      int32_t* c = p.scratch + static_cast<size_t>(w) * G + g;
      const int32_t v = *c;
      *c = r;
      r += v;
    }
  }
}

// Stable placement of every entry; dynamic shared memory: WARPS x G int32.
__global__ void __launch_bounds__(THREADS) bsg_moe_scatter_kernel(const __grid_constant__ Params p) {
  extern __shared__ int32_t moe_smem[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int w = blockIdx.x * WARPS + wib;
  dependency_wait();                                     // the scan kernel's positions are complete
  // the unused tail [placed, n): -1 in both expanded maps (grid-stride over the whole grid)
  {
    const long long placed = __ldg(p.expert_offsets + p.G);
    const long long stride = static_cast<long long>(gridDim.x) * THREADS;
    for (long long q = placed + static_cast<long long>(blockIdx.x) * THREADS + threadIdx.x; q < p.n; q += stride) {
      p.src_rows[q] = -1;
      p.m_indices[q] = -1;
    }
  }
  if (w >= p.tiles) return;                              // warp-uniform
  int32_t* row = moe_smem + static_cast<size_t>(wib) * p.G;
  const int32_t* start = p.scratch + static_cast<size_t>(w) * p.G;
  for (int g = lane; g < p.G; g += 32) row[g] = start[g];
  __syncwarp();
  const int i0 = w * p.tile;
  const int i1 = static_cast<int>(min(p.n, static_cast<long long>(i0) + p.tile));
  const unsigned top_k = static_cast<unsigned>(p.top_k);
  const unsigned lt = (1u << lane) - 1u;
  for (int base = i0; base < i1; base += 32 * BATCH) {
    int32_t g[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int i = base + 32 * j + lane;
      g[j] = i < i1 ? expert_at(p, i) : -1;
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int i = base + 32 * j + lane;
      const unsigned peers = __match_any_sync(0xffffffffu, g[j]);
      const int leader = __ffs(peers) - 1;
      int32_t pos0 = 0;
      if (g[j] >= 0 && lane == leader) {
        pos0 = row[g[j]];
        row[g[j]] = pos0 + __popc(peers);
      }
      pos0 = __shfl_sync(0xffffffffu, pos0, leader);
      __syncwarp();
      if (i < i1) {
        if (g[j] >= 0) {
          const int32_t pos = pos0 + __popc(peers & lt);
          p.src_rows[pos] = static_cast<int32_t>(static_cast<unsigned>(i) / top_k);
          p.m_indices[pos] = g[j];
          p.dst_rows[i] = pos;
        } else {
          p.dst_rows[i] = -1;
        }
      }
    }
  }
}

// The whole permutation in one CTA of FUSED_THREADS threads (n <= FUSED_MAX_N, G <= FUSED_MAX_G, tile a
// multiple of 32 with FUSED_WARPS tiles covering n).  Dynamic shared memory: FUSED_WARPS x G int32.
__global__ void __launch_bounds__(FUSED_THREADS) bsg_moe_fused_kernel(const __grid_constant__ Params p) {
  extern __shared__ int32_t moe_smem[];
  __shared__ int32_t warp_incl[FUSED_WARPS];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int w = tid >> 5;
  const int G = p.G;
  const int n = static_cast<int>(p.n);
  const unsigned top_k = static_cast<unsigned>(p.top_k);
  for (int j = tid; j < FUSED_WARPS * G; j += FUSED_THREADS) moe_smem[j] = 0;
  __syncthreads();
  int32_t* row = moe_smem + w * G;
  const int i0 = w * p.tile;                   // every warp takes part in the barriers, tile or not
  const int i1 = min(n, i0 + p.tile);
  // 1. counts of this warp's tile
  for (int base = i0; base < i1; base += 32 * BATCH) {
    int32_t g[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int i = base + 32 * j + lane;
      g[j] = i < i1 ? expert_at(p, i) : -1;
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const unsigned peers = __match_any_sync(0xffffffffu, g[j]);
      if (g[j] >= 0 && lane == __ffs(peers) - 1) row[g[j]] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  // 2. thread e owns expert e: its total over the tiles, the exclusive scan over experts, then the
  // running sum down the tiles in place of the counts
  int32_t total = 0;
  if (tid < G)
    for (int v = 0; v < FUSED_WARPS; ++v) total += moe_smem[v * G + tid];
  int32_t incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_incl[w] = incl;
  __syncthreads();
  if (w == 0) {
    int32_t t = warp_incl[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t += u;
    }
    warp_incl[lane] = t;
  }
  __syncthreads();
  const int32_t placed = warp_incl[FUSED_WARPS - 1];
  if (tid < G) {
    int32_t r = incl - total + (w > 0 ? warp_incl[w - 1] : 0);
    p.expert_offsets[tid] = r;
    for (int v = 0; v < FUSED_WARPS; ++v) {
      const int32_t c = moe_smem[v * G + tid];
      moe_smem[v * G + tid] = r;
      r += c;
    }
  }
  if (tid == 0) p.expert_offsets[G] = placed;
  __syncthreads();
  // 3. stable placement, as in bsg_moe_scatter_kernel
  const unsigned lt = (1u << lane) - 1u;
  for (int base = i0; base < i1; base += 32 * BATCH) {
    int32_t g[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int i = base + 32 * j + lane;
      g[j] = i < i1 ? expert_at(p, i) : -1;
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int i = base + 32 * j + lane;
      const unsigned peers = __match_any_sync(0xffffffffu, g[j]);
      const int leader = __ffs(peers) - 1;
      int32_t pos0 = 0;
      if (g[j] >= 0 && lane == leader) {
        pos0 = row[g[j]];
        row[g[j]] = pos0 + __popc(peers);
      }
      pos0 = __shfl_sync(0xffffffffu, pos0, leader);
      __syncwarp();
      if (i < i1) {
        if (g[j] >= 0) {
          const int32_t pos = pos0 + __popc(peers & lt);
          p.src_rows[pos] = static_cast<int32_t>(static_cast<unsigned>(i) / top_k);
          p.m_indices[pos] = g[j];
          p.dst_rows[i] = pos;
        } else {
          p.dst_rows[i] = -1;
        }
      }
    }
  }
  for (int q = placed + tid; q < n; q += FUSED_THREADS) {
    p.src_rows[q] = -1;
    p.m_indices[q] = -1;
  }
}

}  // namespace moe
}  // namespace bsg
