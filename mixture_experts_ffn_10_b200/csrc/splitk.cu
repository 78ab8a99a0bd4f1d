// splitk.cu -- the split-K factor of the bf16 tensor-core GEMMs when they have fewer
// tiles than SMs (small token counts: every SM should stream weights).
//
// The GEMM then writes each split's fp32 partial accumulators; the last split of a
// tile region to finish adds them in split order (so the result does not depend on
// timing) and applies the same epilogue as the unsplit GEMM (gemm_tc.cu).
#include "common.cuh"

namespace moe {

// Cost of a split factor in 64-deep K steps per CTA: the waves of work units
// times (K steps per unit + kUnitOverhead for a unit's pipeline fill and
// epilogue), plus kReduceCost for the last split's read-back of the partials
// when S > 1.
constexpr int64_t kUnitOverhead = 2;
constexpr int64_t kReduceCost = 4;

int choose_splits(int64_t tiles, int nkb, int sms) {
  if (tiles <= 0 || tiles >= sms) return 1;
  int best = 1;
  int64_t best_cost = ((tiles + sms - 1) / sms) * (nkb + kUnitOverhead);
  for (int s = 2; s <= 8 && 2 * s <= nkb; s++) {
    const int64_t cost = ((tiles * s + sms - 1) / sms) * ((nkb + s - 1) / s + kUnitOverhead) + kReduceCost;
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

}  // namespace moe
