// Non-uniform per-head budgets from sensitivity curves by greedy swaps
// ("Fast KV Compaction via Attention Matching": zhichai.net/en summary,
// "Engineering Practicality" (sensitivity curves rank the heads once; a
// greedy-swap algorithm assigns the per-head ratios); zhichai.net deep dive
// §4.2 steps 1-2).  Host code: a once-per-model calibration, no GPU work.
//
// loss[h][g] is head h's loss at budget t_min + g·quantum.  The levels start
// as even as the total allows; each swap moves one quantum from the head
// that loses least by giving it up (the donor, never the receiver) to the
// head that gains most by receiving it, ties to the lower head, for as long
// as the gain exceeds the cost.  Every swap lowers the summed loss, so the
// loop ends; with convex curves the result minimises the summed loss.
#include "am_b200.h"

#include <math.h>

#include <vector>

extern "C" am_status_t am_assign_budgets(const double* loss, int32_t num_heads, int32_t levels, int32_t t_min,
                                         int32_t quantum, int64_t total, int32_t max_swaps,
                                         int32_t* budgets_out, int32_t* swaps_out) {
  if (!loss || !budgets_out) return AM_ERR_INVALID_ARG;
  if (num_heads < 1 || levels < 1 || t_min < 1 || quantum < 1) return AM_ERR_INVALID_ARG;
  const int H = num_heads, G = levels;
  for (int64_t e = 0; e < (int64_t)H * G; ++e)
    if (!isfinite(loss[e])) return AM_ERR_NONFINITE;
  const int64_t rest = total - (int64_t)H * t_min;
  if (rest < 0 || rest % quantum != 0 || rest / quantum > (int64_t)H * (G - 1)) return AM_ERR_BUDGET;
  if ((int64_t)t_min + (int64_t)quantum * (G - 1) > 0x7fffffffll) return AM_ERR_UNSUPPORTED;
  const int64_t units = rest / quantum;
  std::vector<int> lev(H);
  for (int h = 0; h < H; ++h) lev[h] = (int)(units / H + (h < units % H ? 1 : 0));
  int swaps = 0;
  while (max_swaps < 0 || swaps < max_swaps) {
    int b = -1;
    double gain = -INFINITY;
    for (int h = 0; h < H; ++h) {
      if (lev[h] < G - 1) {
        const double gh = loss[(int64_t)h * G + lev[h]] - loss[(int64_t)h * G + lev[h] + 1];
        if (gh > gain) { b = h; gain = gh; }
      }
    }
    int a = -1;
    double cost = INFINITY;
    for (int h = 0; h < H; ++h) {
      if (h != b && lev[h] > 0) {
        const double ch = loss[(int64_t)h * G + lev[h] - 1] - loss[(int64_t)h * G + lev[h]];
        if (ch < cost) { a = h; cost = ch; }
      }
    }
    if (a < 0 || b < 0 || !(gain > cost)) break;
    --lev[a];
    ++lev[b];
    ++swaps;
  }
  for (int h = 0; h < H; ++h) budgets_out[h] = t_min + quantum * lev[h];
  if (swaps_out) *swaps_out = swaps;
  return AM_OK;
}
