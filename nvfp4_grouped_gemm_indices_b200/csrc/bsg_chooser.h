// bsg_chooser.h -- tactic table, score and overrides (host only).
#pragma once
#include <cstdint>

// Grid override for tests of the persistent schedule (bsg_set_max_ctas); returns `grid` when unset.
int bsg_forced_grid(int kind, int grid);

// Work-unit estimates the score uses (from sizes only; m_indices stays on the device).
struct BsgUnitEstimate {
  int64_t windows;    // ceil(M / 128)
  int64_t segments;   // window segments: windows + (runs - 1), runs <= min(G, M)
  int64_t pairs;      // expected pairs of same-expert segments (2-SM tiles): runs * ceil(span / 2)
  int64_t pairs_max;  // upper bound on the pairs the scheduler can form (sizes the SM-pair grid)
};
BsgUnitEstimate bsg_estimate_units(int64_t M, int64_t G);

// Measured winners (bsg_autotune_*) for exact problem sizes; bsg_choose_tactic prefers them to the
// score.  bsg_tuned_tactic returns -1 when the sizes were never tuned.
void bsg_record_tuned(int kind, int64_t M, int64_t N, int64_t K, int64_t G, int tactic);
int bsg_tuned_tactic(int kind, int64_t M, int64_t N, int64_t K, int64_t G);

