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
//               tiles (the scratch row of tile w now holds where w's entries of each expert begin).
//   3. scatter: each warp walks its tile again in order with its row of starting positions in
//               shared memory; an entry's position is its group's base plus its rank among the
//               group's lanes, and the group's first lane advances the base -- so entries of one
//               expert keep their token order (stable) inside a tile, across tiles by the scan.
//               The kernel also fills the unused tail positions with -1.
// The counting is integer work bound by the latency of its dependent steps, not by a roofline; all
// memory traffic is coalesced except the scattered 4-byte output writes.
#pragma once

#include <cstdint>

namespace bsg {
namespace moe {

constexpr int WARPS = 4;                 // warps (tiles) per CTA of the count and scatter kernels
constexpr int THREADS = WARPS * 32;
constexpr int SCAN_THREADS = 1024;
constexpr int MIN_TILE = 256;            // entries per tile when the scratch allows it

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
  if (w >= p.tiles) return;                              // warp-uniform
  for (int g = lane; g < p.G; g += 32) row[g] = 0;
  __syncwarp();
  const long long i0 = static_cast<long long>(w) * p.tile;
  const long long i1 = min(p.n, i0 + p.tile);
  for (long long base = i0; base < i1; base += 32) {
    const long long i = base + lane;
    const int32_t g = i < i1 ? expert_at(p, i) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, g);
    if (g >= 0 && lane == __ffs(peers) - 1) row[g] += __popc(peers);
    __syncwarp();
  }
  int32_t* out = p.scratch + static_cast<size_t>(w) * p.G;
  for (int g = lane; g < p.G; g += 32) out[g] = row[g];
}

// One CTA: expert_offsets (exclusive scan over experts of the per-expert totals) and, in place of
// each tile's counts, the position where that tile's entries of each expert begin.  Dynamic shared
// memory: G int32 (the totals, then the offsets).
__global__ void __launch_bounds__(SCAN_THREADS) bsg_moe_scan_kernel(const __grid_constant__ Params p) {
  extern __shared__ int32_t moe_smem[];
  __shared__ int32_t part[SCAN_THREADS];
  const int tid = threadIdx.x;
  for (int g = tid; g < p.G; g += SCAN_THREADS) {
    int32_t sum = 0;
    int w = 0;
    for (; w + 8 <= p.tiles; w += 8) {                   // eight independent loads in flight
      int32_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = p.scratch[static_cast<size_t>(w + j) * p.G + g];
#pragma unroll
      for (int j = 0; j < 8; ++j) sum += v[j];
    }
    for (; w < p.tiles; ++w) sum += p.scratch[static_cast<size_t>(w) * p.G + g];
    moe_smem[g] = sum;
  }
  __syncthreads();
  // exclusive scan of moe_smem[0, G): thread tid owns the consecutive experts [tid * per, +per)
  const int per = (p.G + SCAN_THREADS - 1) / SCAN_THREADS;
  const int g0 = tid * per;
  int32_t local = 0;
  for (int j = 0; j < per && g0 + j < p.G; ++j) local += moe_smem[g0 + j];
  part[tid] = local;
  __syncthreads();
  for (int off = 1; off < SCAN_THREADS; off <<= 1) {     // inclusive Hillis-Steele scan of part[]
    const int32_t v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int32_t run = part[tid] - local;                       // exclusive prefix of this thread's experts
  for (int j = 0; j < per && g0 + j < p.G; ++j) {
    const int32_t c = moe_smem[g0 + j];
    moe_smem[g0 + j] = run;
    p.expert_offsets[g0 + j] = run;
    run += c;
  }
  if (tid == SCAN_THREADS - 1) p.expert_offsets[p.G] = part[SCAN_THREADS - 1];
  __syncthreads();
  for (int g = tid; g < p.G; g += SCAN_THREADS) {
    int32_t r = moe_smem[g];
    int w = 0;
    for (; w + 8 <= p.tiles; w += 8) {
      int32_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = p.scratch[static_cast<size_t>(w + j) * p.G + g];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        p.scratch[static_cast<size_t>(w + j) * p.G + g] = r;
        r += v[j];
      }
    }
    for (; w < p.tiles; ++w) {
      int32_t* c = p.scratch + static_cast<size_t>(w) * p.G + g;
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
  const long long i0 = static_cast<long long>(w) * p.tile;
  const long long i1 = min(p.n, i0 + p.tile);
  const unsigned lt = (1u << lane) - 1u;
  for (long long base = i0; base < i1; base += 32) {
    const long long i = base + lane;
    const bool in = i < i1;
    const int32_t g = in ? expert_at(p, i) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, g);
    const int leader = __ffs(peers) - 1;
    int32_t pos0 = 0;
    if (g >= 0 && lane == leader) {
      pos0 = row[g];
      row[g] = pos0 + __popc(peers);
    }
    pos0 = __shfl_sync(0xffffffffu, pos0, leader);
    __syncwarp();
    if (in) {
      if (g >= 0) {
        const int32_t pos = pos0 + __popc(peers & lt);
        p.src_rows[pos] = static_cast<int32_t>(i / p.top_k);
        p.m_indices[pos] = g;
        p.dst_rows[i] = pos;
      } else {
        p.dst_rows[i] = -1;
      }
    }
  }
}

}  // namespace moe
}  // namespace bsg
