// bsg_chooser.h -- tactic table, score and overrides (host only).
#pragma once
#include <cstdint>

// Grid override for tests of the persistent schedule (bsg_set_max_ctas); returns `grid` when unset.
int bsg_forced_grid(int kind, int grid);

// Work-unit estimates the score uses (from sizes only; m_indices stays on the device).
struct BsgUnitEstimate {
  int64_t windows;    // ceil(M / 128)
  int64_t segments;   // window segments: windows + (runs - 1), runs <= min(G, M)
  int64_t pairs;      // pairs of same-expert segments (2-SM tiles)
};
BsgUnitEstimate bsg_estimate_units(int64_t M, int64_t G);
