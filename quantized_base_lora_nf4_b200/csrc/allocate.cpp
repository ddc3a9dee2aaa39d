// LQ-LoRA's budgeted choice of quantisation parameters per matrix (LQ-LoRA abstract: an integer linear
// programme picks each matrix's bit width and block size so that the whole model meets a memory
// budget).  A multiple-choice knapsack: each matrix takes one option, the summed reconstruction error
// is minimised and the summed storage stays within the budget.  Host code; exact dynamic programming
// over the budget in whole units (costs rounded up, so a plan never exceeds the budget).
#include <cstdint>
#include <limits>
#include <vector>

#include "../../include/qlr.h"

extern "C" int qlr_lqlora_allocate(const double* err, const int64_t* cost_bits, int n_mat, int n_opt,
                                   int64_t budget_bits, int64_t unit_bits, int* choice, double* total_err) {
  if (!err || !cost_bits || !choice || n_mat <= 0 || n_opt <= 0 || n_opt > 255 || unit_bits <= 0 || budget_bits < 0)
    return QLR_ERR_ARG;
  const int64_t B = budget_bits / unit_bits;
  if ((B + 1) * static_cast<int64_t>(n_mat) > (int64_t(1) << 30)) return QLR_ERR_SHAPE;  // choose a larger unit
  std::vector<int64_t> units(static_cast<size_t>(n_mat) * n_opt);
  for (size_t e = 0; e < units.size(); ++e) {
    if (cost_bits[e] < 0) return QLR_ERR_ARG;
    units[e] = (cost_bits[e] + unit_bits - 1) / unit_bits;
  }
  const double inf = std::numeric_limits<double>::infinity();
  std::vector<double> best(static_cast<size_t>(B + 1), 0.0), next(static_cast<size_t>(B + 1));
  std::vector<uint8_t> pick(static_cast<size_t>(n_mat) * (B + 1));
  for (int i = 0; i < n_mat; ++i) {
    const double* e = err + static_cast<size_t>(i) * n_opt;
    const int64_t* u = units.data() + static_cast<size_t>(i) * n_opt;
    uint8_t* p = pick.data() + static_cast<size_t>(i) * (B + 1);
    for (int64_t b = 0; b <= B; ++b) {
      double cur = inf;
      int arg = 0;
      for (int o = 0; o < n_opt; ++o) {  // the first minimum over the options
        if (u[o] <= b) {
          const double v = best[static_cast<size_t>(b - u[o])] + e[o];
          if (v < cur) {
            cur = v;
            arg = o;
          }
        }
      }
      next[static_cast<size_t>(b)] = cur;
      p[b] = static_cast<uint8_t>(arg);
    }
    best.swap(next);
  }
  if (!(best[static_cast<size_t>(B)] < inf)) return QLR_ERR_SHAPE;  // the budget is below the cheapest plan
  int64_t b = B;
  for (int i = n_mat - 1; i >= 0; --i) {  // read the plan back from the full budget, last matrix first
    const int o = pick[static_cast<size_t>(i) * (B + 1) + b];
    choice[i] = o;
    b -= units[static_cast<size_t>(i) * n_opt + o];
  }
  if (total_err) *total_err = best[static_cast<size_t>(B)];
  return QLR_OK;
}
