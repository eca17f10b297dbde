// bsg_chooser.h -- tactic table, score and overrides (host only).
#pragma once
#include <cstdint>

// Grid override for tests of the persistent schedule (bsg_set_max_ctas); returns `grid` when unset.
int bsg_forced_grid(int kind, int grid);
