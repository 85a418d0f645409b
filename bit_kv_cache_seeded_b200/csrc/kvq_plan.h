// Split plan of the decode kernels: how many CTAs share one (sequence, kv-head) row of the cache
// and how many tokens each takes. Plain C++ (no CUDA types), so host tests compile it alone.
//
// A split covers a whole number of 64-token units (two cache tiles), at most `max_units` of them.
// plan_splits picks the split count that minimises waves x (units per CTA + a fixed per-CTA
// overhead of 4 units), a wave holding slots_per_sm(units per CTA) resident CTAs on each of `sms`
// SMs; chunks may be as small as half the largest (smaller chunks need less shared memory for their
// logits, so more CTAs can be resident). max_splits bounds the split count for every length up to
// the capacity: the workspace is sized from it once, so no call may plan more splits than it returns.
#pragma once

#include <algorithm>

namespace kvq {

constexpr int kPlanUnitTokens = 64;  // tokens of one split unit
constexpr int kPlanUnitTiles = 2;    // cache tiles of one split unit

inline int min_plan_units(int max_units) { return std::max(1, max_units / 2); }

inline int max_splits(int pairs, int sms, int tiles, int max_units, int waves_bound) {
  const int units = std::max(1, tiles / kPlanUnitTiles);
  const int need = (units + min_plan_units(max_units) - 1) / min_plan_units(max_units);
  const int bound = std::max(1, (waves_bound * sms + pairs - 1) / pairs);
  return std::max(need, std::min(bound, units));
}

template <class SlotsFn>
void plan_splits(int pairs, int sms, const SlotsFn& slots_per_sm, int max_units, int waves_bound, int max_len,
                 int* splits, int* chunk) {
  const int units = std::max(1, (max_len + kPlanUnitTokens - 1) / kPlanUnitTokens);
  const int smin = (units + max_units - 1) / max_units;
  const int smax = std::min(max_splits(pairs, sms, units * kPlanUnitTiles, max_units, waves_bound), units);
  long best_cost = -1;
  int best_cu = units;
  for (int s = std::max(1, smin); s <= std::max(smin, smax); ++s) {
    const int cu = (units + s - 1) / s;
    if (cu > max_units) continue;
    const int ss = (units + cu - 1) / cu;
    const long slots = (long)sms * slots_per_sm(cu);
    const long waves = ((long)pairs * ss + slots - 1) / slots;
    const long cost = waves * (cu + 4);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_cu = cu; }
  }
  *splits = (units + best_cu - 1) / best_cu;
  *chunk = best_cu * kPlanUnitTokens;
}

}  // namespace kvq
