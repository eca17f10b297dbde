// bsg_sched.cuh -- the expert-run-aware window scheduler shared by both kernels.
//
// The rows of A are cut into 128-row windows [128w, 128w + 128).  Inside a window every maximal
// stretch of consecutive rows routed to the same expert is one *segment* (row_lo, row_hi, g); rows
// routed nowhere (index < 0 or >= G) belong to no segment.  A *work unit* is (segment, N tile).  The
// tile always covers the whole window (TMA loads the 128 rows starting at 128w, zero-filling past M),
// and the epilogue writes only the segment's rows: rows are masked, never padded or gathered.
// This is the window-segment program of the page "[flashinfer] FlashInfer FP8 GEMM 최적화: 윈도우
// 세그먼트 KG1 프로그램으로 GPU 성능 극대화", section 2 (one CTA per expert run inside a window,
// m_indices re-read on every call so CUDA-graph replays see new routings), made persistent: the
// units are numbered window by window, segment by segment, N tile by N tile, and CTA b of a grid of
// P takes units b, b + P, b + 2P, ...  A dedicated scheduler warp walks the windows, finds the
// segments with warp ballots and hands the CTA's units to the other roles through a small
// shared-memory queue guarded by mbarriers.
#pragma once

#include "bsg_ptx.cuh"

namespace bsg {

struct Unit {
  int row0;    // first row of the window (multiple of 128)
  int row_lo;  // segment rows [row_lo, row_hi), all routed to expert g
  int row_hi;
  int g;
  int n0;      // first output column of the tile
  int valid;   // 0 = no more units for this CTA
  int pad0, pad1;
};

template <int Q>
struct UnitQueue {
  Unit slot[Q];
  uint64_t full[Q];
  uint64_t empty[Q];
};

struct WaitCtx {
  uint64_t timeout_ns;
  volatile int* abort;
  DeviceStatus* status;
};

// Ring position (stage, phase) advanced at every use; carried across work units.
template <int STAGES>
struct RingPos {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++stage == STAGES) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// On an aborted run a producer must not retire while its TMA loads are still landing in shared
// memory.  The loads of the last min(issued, STAGES) uses of the ring may be in flight; each of those
// uses completes its own transaction barrier (`bars`) when the bytes have arrived, independently of
// every other role, so this bounded wait (which ignores the abort flag) ends by itself.
template <int STAGES>
__device__ __forceinline__ void drain_inflight_loads(uint64_t* bars, RingPos<STAGES> pos, long long issued,
                                                     const WaitCtx& w) {
  const int n = issued < STAGES ? static_cast<int>(issued) : STAGES;
  for (int i = 0; i < n; ++i) {
    // step back one use
    if (pos.stage == 0) {
      pos.stage = STAGES - 1;
      pos.phase ^= 1u;
    } else {
      --pos.stage;
    }
    mbar_wait(&bars[pos.stage], pos.phase, w.timeout_ns, nullptr, nullptr, kSiteDrain, pos.stage);
  }
}

// Debug fault injection (test only): the scheduler hands out no unit and no end marker, so every
// other role's bounded wait on the unit queue expires; no memory operation is ever issued.
constexpr int kDebugWithholdSchedule = 1;

// Consumer side: returns false on abort/timeout.  `u` receives the unit (u.valid == 0: done).
template <int Q>
__device__ __forceinline__ bool queue_pop(UnitQueue<Q>& q, int& slot, uint32_t& phase, Unit& u,
                                          const WaitCtx& w) {
  if (!mbar_wait(&q.full[slot], phase, w.timeout_ns, w.abort, w.status, kSiteQueueFull, slot)) return false;
  u = q.slot[slot];
  __syncwarp();
  if (lane_idx() == 0) mbar_arrive(&q.empty[slot]);
  if (++slot == Q) {
    slot = 0;
    phase ^= 1u;
  }
  return true;
}

template <int Q>
__device__ __forceinline__ bool queue_push(UnitQueue<Q>& q, int& slot, uint32_t& phase, const Unit& u,
                                           const WaitCtx& w) {
  if (!mbar_wait(&q.empty[slot], phase ^ 1u, w.timeout_ns, w.abort, w.status, kSiteQueueEmpty, slot))
    return false;
  if (lane_idx() == 0) {
    q.slot[slot] = u;
    mbar_arrive(&q.full[slot]);
  }
  __syncwarp();
  if (++slot == Q) {
    slot = 0;
    phase ^= 1u;
  }
  return true;
}

__device__ __forceinline__ int routed_expert(const int* __restrict__ m_indices, int row, int M, int G) {
  if (row >= M) return -1;
  int g = m_indices ? __ldg(m_indices + row) : 0;
  return (g >= 0 && g < G) ? g : -1;
}

// Scheduler warp body.  n_tiles = ceil(N / BN); n_group = N tiles per raster group.
//
// Unit order: for each group of n_group consecutive N tiles, for each window, for each segment of
// the window, for each N tile of the group.  With n_group = n_tiles this is window-major (the rows
// of a window are reused from L2 across all N tiles, and B[g] across the windows of an expert);
// smaller groups keep a slice of a large B resident while all windows stream past it.
// The m_indices of kScanBatch windows are loaded at once, so walking to a CTA's first unit costs
// one memory latency per kScanBatch windows.
//
// PAIR = false: one CTA per unit; CTA b of P takes units b, b + P, ...
// PAIR = true : two CTAs (a cluster pair) per unit.  Consecutive segments (in window order) of the
// same expert are paired -- a run spanning several windows gives pairs of consecutive windows -- and
// a segment without a partner is paired with an empty half (rows [0, 0): computed, never stored).
// Cluster c of P/2 takes pair-units c, c + P/2, ...; CTA rank r of the pair receives half r.
// TOK < 128 (PAIR = false only): a segment longer than TOK rows is cut into consecutive chunks of at
// most TOK rows, each its own row tile (the operand-swapped kernel, whose token tile is TOK wide).
constexpr int kScanBatch = 4;

struct Seg {
  int row0, lo, hi, g;
};

template <int Q, int BN, bool PAIR, int TOK = 128>
__device__ void run_scheduler(UnitQueue<Q>& q, const int* __restrict__ m_indices, int M, int G, int n_tiles,
                              int n_group, const WaitCtx& wctx, int debug_mode) {
  if (debug_mode == kDebugWithholdSchedule) return;
  const int lane = lane_idx();
  const unsigned FULL = 0xffffffffu;
  int slot = 0;
  uint32_t phase = 0;
  const long long owner = PAIR ? blockIdx.x / 2 : blockIdx.x;   // cluster (pair) or CTA index
  const long long stride = PAIR ? gridDim.x / 2 : gridDim.x;
  const int half = PAIR ? static_cast<int>(blockIdx.x & 1) : 0;
  long long next = owner;                 // next global unit index this CTA (pair) owns
  long long first = 0;                    // global index of the first unit of the next segment/pair
  const int n_windows = (M + 127) / 128;
  const int n_groups = (n_tiles + n_group - 1) / n_group;
  bool alive = true;

  // hand out the units [first, first + tiles) that this CTA owns; returns false on abort
  auto emit = [&](const Seg& a, const Seg* b, int t0, int tiles) -> bool {
    const long long base = first;
    first += tiles;
    if (next >= base + tiles) return true;
    Unit u;
    const Seg* mine = (half == 0) ? &a : b;
    if (mine) {
      u.row0 = mine->row0;
      u.row_lo = mine->lo;
      u.row_hi = mine->hi;
    } else {
      u.row0 = a.row0;  // empty half: load the partner's window, store nothing
      u.row_lo = 0;
      u.row_hi = 0;
    }
    u.g = a.g;
    u.valid = 1;
    u.pad0 = u.pad1 = 0;
    while (next < base + tiles) {
      u.n0 = (t0 + static_cast<int>(next - base)) * BN;
      if (!queue_push(q, slot, phase, u, wctx)) return false;
      next += stride;
    }
    return true;
  };

  for (int grp = 0; grp < n_groups && alive; ++grp) {
    const int t0 = grp * n_group;
    const int tiles = min(n_group, n_tiles - t0);
    Seg pending;
    bool have_pending = false;
    for (int wb = 0; wb < n_windows && alive; wb += kScanBatch) {
      int gv[kScanBatch][4];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) gv[i][j] = routed_expert(m_indices, (wb + i) * 128 + 32 * j + lane, M, G);
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) {
        const int w = wb + i;
        if (w >= n_windows || !alive) break;
        const int row0 = w * 128;
        uint32_t smask[4], emask[4];
        int nseg = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int prev = __shfl_up_sync(FULL, gv[i][j], 1);
          int nxt = __shfl_down_sync(FULL, gv[i][j], 1);
          const int prev_chunk_last = __shfl_sync(FULL, gv[i][j > 0 ? j - 1 : 0], 31);
          const int next_chunk_first = __shfl_sync(FULL, gv[i][j < 3 ? j + 1 : 3], 0);
          if (lane == 0) prev = (j > 0) ? prev_chunk_last : -1;
          if (lane == 31) nxt = (j < 3) ? next_chunk_first : -1;
          const bool is_start = gv[i][j] >= 0 && gv[i][j] != prev;
          const bool is_end = gv[i][j] >= 0 && gv[i][j] != nxt;
          smask[j] = __ballot_sync(FULL, is_start);
          emask[j] = __ballot_sync(FULL, is_end);
          nseg += __popc(smask[j]);
        }
        if (!PAIR && TOK >= 128) {
          // every segment is a unit: skip the window in one step when this CTA owns none of it
          const long long units_here = static_cast<long long>(nseg) * tiles;
          if (next >= first + units_here) {
            first += units_here;
            continue;
          }
        }
        int js = 0, je = 0;
        uint32_t ms = smask[0], me = emask[0];
        for (int k = 0; k < nseg; ++k) {
          while (ms == 0) { ++js; ms = smask[js]; }
          while (me == 0) { ++je; me = emask[je]; }
          const int bs = __ffs(ms) - 1;
          const int be = __ffs(me) - 1;
          ms &= ms - 1;
          me &= me - 1;
          const int gsel = js == 0 ? gv[i][0] : js == 1 ? gv[i][1] : js == 2 ? gv[i][2] : gv[i][3];
          Seg sg;
          sg.row0 = row0;
          sg.lo = row0 + 32 * js + bs;
          sg.hi = row0 + 32 * je + be + 1;
          sg.g = __shfl_sync(FULL, gsel, bs);
          if (!PAIR) {
            if constexpr (TOK >= 128) {
              if (!emit(sg, nullptr, t0, tiles)) alive = false;
            } else {
              for (int c = sg.lo; c < sg.hi && alive; c += TOK) {
                Seg part = sg;
                part.lo = c;
                part.hi = min(sg.hi, c + TOK);
                if (!emit(part, nullptr, t0, tiles)) alive = false;
              }
            }
          } else if (have_pending && pending.g == sg.g) {
            if (!emit(pending, &sg, t0, tiles)) alive = false;
            have_pending = false;
          } else {
            if (have_pending && !emit(pending, nullptr, t0, tiles)) alive = false;
            pending = sg;
            have_pending = true;
          }
          if (!alive) break;
        }
      }
    }
    if (PAIR && have_pending && alive) {
      if (!emit(pending, nullptr, t0, tiles)) alive = false;
    }
  }
  if (!alive) return;
  Unit done;
  done.row0 = done.row_lo = done.row_hi = done.g = done.n0 = 0;
  done.valid = 0;
  done.pad0 = done.pad1 = 0;
  queue_push(q, slot, phase, done, wctx);
}

}  // namespace bsg
