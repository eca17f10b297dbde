// bsg_chooser.cpp -- the tile / cluster chooser.
//
// Score of a tactic (the ranking of the page "[flashinfer] FlashInfer의 FP4 GEMM 최적화: 휴리스틱
// 개선과 Autotuning 효율화", section 2):
//     score = m_eff * n_eff * throughput / (num_waves * tile_n)
//     score *= 1.05                 if the tactic issues 2-CTA (cta_group::2) MMAs
//     score *= 0.95^(log2 cga_n)    for a cluster of cga_n CTAs along N (multicast)
// The page names but does not define m_eff, n_eff, throughput and num_waves.  Readings used here:
//     m_eff      = rows / rows computed: M / (segments * 128) for one-SM tiles, M / (pairs * 256)
//                  for SM-pair tiles (window segments are the row tiles of this library, so the
//                  padding they waste is what m_eff measures); segments and pairs are estimated from
//                  M and G (sorted routing), since m_indices stays on the device
//     n_eff      = N / (ceil(N / tile_n) * tile_n)
//     num_waves  = ceil(units / (sm_count / cluster_size))
//     throughput = the tile's sustained fraction of the FP8 / FP4 tensor peak measured on the
//                  prefill workloads (the table below); the exhaustive sweep re-measures it
// Operand-swapped FP8 tactics (swap = 1: B rows are the MMA's 128-row operand, a chunk of at most
// tok tokens its N operand): the row tile is a token chunk,
//     m_eff = M / (chunks * tok),  chunks = segments * ceil(M / segments / tok)
// and tile_n is the unit's width in output columns.  The MMA is 16 * ceil(tokens / 16) wide, but a
// unit's time was measured to depend on its K blocks, not on its token count (the per-K-block work
// of the single issuing thread dominates when the MMAs are small), so m_eff charges the whole chunk.
// The sweep over all tactics is what validates the ranking.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <tuple>

#include "../../include/bsg.h"
#include "bsg_chooser.h"

namespace {

struct Tactic {
  const char* name;
  int tile_m;      // rows per tile; for swap tactics the token chunk (tok)
  int tile_n;
  int cta_group;
  int cga_n;
  double throughput;
  int swap;
};

// FP8 and NVFP4 tactic tables (kind 0 and 1).  Only tactics that exist as kernels are listed.
const Tactic kFp8[] = {
    {"fp8_1sm_m128_n256_s4", 128, 256, 1, 1, 0.47, 0},
    {"fp8_2sm_m256_n256_s6", 256, 256, 2, 1, 0.45, 0},
    {"fp8_swapab_1sm_n128_t128_s6", 128, 128, 1, 1, 0.24, 1},
    {"fp8_swapab_1sm_n256_t64_s5", 64, 256, 1, 1, 0.23, 1},
    {"fp8_1sm_m128_n64_s8", 128, 64, 1, 1, 0.19, 0},
};
const Tactic kNvfp4[] = {
    {"nvfp4_1sm_m128_n256_s4", 128, 256, 1, 1, 0.52, 0},
    {"nvfp4_2sm_m256_n256_s5", 256, 256, 2, 1, 0.58, 0},
};

const Tactic* table(int kind, int* n) {
  if (kind == 0) {
    *n = static_cast<int>(sizeof(kFp8) / sizeof(kFp8[0]));
    return kFp8;
  }
  if (kind == 1) {
    *n = static_cast<int>(sizeof(kNvfp4) / sizeof(kNvfp4[0]));
    return kNvfp4;
  }
  *n = 0;
  return nullptr;
}

std::mutex g_mu;
int g_forced_tactic[2] = {-1, -1};
std::map<std::tuple<int, int64_t, int64_t, int64_t, int64_t>, int> g_tuned;
int g_max_ctas[2] = {0, 0};
bool g_env_read = false;

void read_env() {
  if (g_env_read) return;
  g_env_read = true;
  if (const char* t = std::getenv("BSG_TACTIC")) {
    int v = std::atoi(t);
    g_forced_tactic[0] = g_forced_tactic[1] = v;
  }
}

}  // namespace

BsgUnitEstimate bsg_estimate_units(int64_t M, int64_t G) {
  BsgUnitEstimate e;
  e.windows = (M + 127) / 128;
  const int64_t runs = G < M ? G : M;
  e.segments = e.windows + runs - 1;
  // pairs: the scheduler pairs consecutive segments of one run, so a run cut into s segments gives
  // ceil(s / 2) pairs; with R equal runs each spans ceil(M / (128 R)) windows, plus one more when
  // runs start at arbitrary rows (R > 1)
  const int64_t span = (M + 128 * runs - 1) / (128 * runs) + (runs > 1 ? 1 : 0);
  e.pairs_max = (e.segments + 1) / 2 + runs / 2;
  e.pairs = runs * ((span + 1) / 2);
  if (e.pairs > e.pairs_max) e.pairs = e.pairs_max;
  return e;
}

void bsg_record_tuned(int kind, int64_t M, int64_t N, int64_t K, int64_t G, int tactic) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_tuned[std::make_tuple(kind, M, N, K, G)] = tactic;
}

int bsg_tuned_tactic(int kind, int64_t M, int64_t N, int64_t K, int64_t G) {
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_tuned.find(std::make_tuple(kind, M, N, K, G));
  return it == g_tuned.end() ? -1 : it->second;
}

int bsg_forced_grid(int kind, int grid) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (kind < 0 || kind > 1) return grid;
  int cap = g_max_ctas[kind];
  if (cap > 0 && cap < grid) return cap;
  return grid;
}

extern "C" {

int bsg_num_tactics(int kind) {
  int n = 0;
  table(kind, &n);
  return n;
}

const char* bsg_tactic_name(int kind, int tactic) {
  int n = 0;
  const Tactic* t = table(kind, &n);
  if (!t || tactic < 0 || tactic >= n) return "";
  return t[tactic].name;
}

double bsg_tactic_score(int kind, int tactic, int64_t M, int64_t N, int64_t K, int64_t G, int sm_count) {
  (void)K;
  int n = 0;
  const Tactic* tt = table(kind, &n);
  if (!tt || tactic < 0 || tactic >= n || M <= 0 || N <= 0 || G <= 0 || sm_count <= 0) return 0.0;
  const Tactic& t = tt[tactic];
  const BsgUnitEstimate est = bsg_estimate_units(M, G);
  double row_tiles = static_cast<double>(t.cta_group == 2 ? est.pairs : est.segments);
  const double tiles_n = std::ceil(static_cast<double>(N) / t.tile_n);
  double m_eff = static_cast<double>(M) / (row_tiles * t.tile_m);
  if (t.swap) {
    const double seg = static_cast<double>(est.segments);
    row_tiles = seg * std::ceil(std::ceil(static_cast<double>(M) / seg) / t.tile_m);
    m_eff = static_cast<double>(M) / (row_tiles * t.tile_m);
    if (m_eff > 1.0) m_eff = 1.0;
  }
  const double n_eff = static_cast<double>(N) / (tiles_n * t.tile_n);
  const int cluster = t.cta_group * t.cga_n;
  const double units = row_tiles * tiles_n;
  const double slots = std::floor(static_cast<double>(sm_count) / cluster);
  const double waves = std::ceil(units / (slots > 0 ? slots : 1.0));
  double score = m_eff * n_eff * t.throughput / (waves * t.tile_n);
  if (t.cta_group == 2) score *= 1.05;
  int bits = 0;
  for (int v = t.cga_n; v > 1; v >>= 1) ++bits;
  score *= std::pow(0.95, bits);
  return score;
}

int bsg_choose_tactic(int kind, int64_t M, int64_t N, int64_t K, int64_t G, int sm_count) {
  int n = 0;
  if (!table(kind, &n)) return BSG_ERR_INVALID_ARG;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    read_env();
    int f = g_forced_tactic[kind];
    if (f >= 0 && f < n) return f;
    auto it = g_tuned.find(std::make_tuple(kind, M, N, K, G));
    if (it != g_tuned.end() && it->second >= 0 && it->second < n) return it->second;
  }
  int best = 0;
  double best_score = -1.0;
  for (int i = 0; i < n; ++i) {
    double sc = bsg_tactic_score(kind, i, M, N, K, G, sm_count);
    if (sc > best_score) {
      best_score = sc;
      best = i;
    }
  }
  return best;
}

bsg_status bsg_set_tactic(int kind, int tactic) {
  int n = 0;
  if (!table(kind, &n)) return BSG_ERR_INVALID_ARG;
  if (tactic >= n) return BSG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  read_env();
  g_forced_tactic[kind] = tactic < 0 ? -1 : tactic;
  return BSG_OK;
}

void bsg_autotune_clear(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_tuned.clear();
}

bsg_status bsg_set_max_ctas(int kind, int max_ctas) {
  if (kind < 0 || kind > 1 || max_ctas < 0) return BSG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  g_max_ctas[kind] = max_ctas;
  return BSG_OK;
}

}  // extern "C"
