// lr_gac.cu — host code: GAC's re-selection of compressed dimensions under
// a parameter budget ("Why Smaller Is Slower? Dimensional Misalignment in
// Compressed LLMs", §4.3 Step 3: Constrained Optimization, with its budget
// quantization).  Nothing here touches the GPU.
//
// Weight i keeps one of its candidate dimensions (the aligned, cliff-free
// sizes its dimension sweep, §4.2, produced); candidate j stores w_ij
// parameters.  The selection maximises Σ_i s_i·(w_ij − |W_i*|) — importance
// times the parameters kept beyond (or short of) the unconstrained
// allocation |W_i*| — subject to Σ_i w_ij fitting the budget B.  It is a
// multiple-choice knapsack, solved by the recurrence
//     D[i][b] = max_j D[i−1][b − w'_ij] + v_ij,   D[0][b] = 0,
// over quantized costs w'_ij = ⌈w_ij / u⌉ and budget B' = ⌊B / u⌋, so that
// D[n][B'] is the best selection whose quantized cost is at most B'.
// Rounding costs up and the budget down keeps every selection within B.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <new>
#include <utility>
#include <vector>

#include "lr_linear.h"

namespace {

constexpr int kMaxCandidates = 255;             // the argmax table holds one byte
constexpr int64_t kMaxParams = int64_t(1) << 53;  // costs convert to double exactly
constexpr int64_t kMaxTableBytes = int64_t(1) << 30;

}  // namespace

extern "C" lr_status lr_gac_select(int n_items, const int* n_cand, const int64_t* cost,
                                   const double* score, const int64_t* base, int64_t budget,
                                   int64_t unit, int* choice, double* objective) {
  if (n_items < 1 || !n_cand || !cost || !score || !base || !choice || budget < 0 || unit < 1)
    return LR_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int i = 0; i < n_items; ++i) {
    if (n_cand[i] < 1 || n_cand[i] > kMaxCandidates) return LR_ERR_INVALID_ARG;
    if (!std::isfinite(score[i]) || base[i] < 0 || base[i] > kMaxParams) return LR_ERR_INVALID_ARG;
    total += n_cand[i];
  }
  const int64_t bq = budget / unit;
  if (bq >= kMaxTableBytes / n_items) return LR_ERR_UNSUPPORTED;
  try {
    // Quantized costs and the values v_ij = s_i·(w_ij − |W_i*|).
    std::vector<int64_t> wq(static_cast<size_t>(total));
    std::vector<double> val(static_cast<size_t>(total));
    int64_t off = 0;
    for (int i = 0; i < n_items; ++i) {
      for (int j = 0; j < n_cand[i]; ++j, ++off) {
        const int64_t w = cost[off];
        if (w < 0 || w > kMaxParams) return LR_ERR_INVALID_ARG;
        wq[off] = w / unit + (w % unit != 0 ? 1 : 0);
        val[off] = score[i] * static_cast<double>(w - base[i]);
        if (!std::isfinite(val[off])) return LR_ERR_INVALID_ARG;
      }
    }
    const size_t width = static_cast<size_t>(bq) + 1;
    const double ninf = -std::numeric_limits<double>::infinity();
    std::vector<uint8_t> arg(static_cast<size_t>(n_items) * width);
    std::vector<double> prev(width, 0.0), cur(width);
    off = 0;
    for (int i = 0; i < n_items; ++i) {
      uint8_t* ai = arg.data() + static_cast<size_t>(i) * width;
      std::fill(cur.begin(), cur.end(), ninf);
      std::fill(ai, ai + width, uint8_t{0});
      // Candidates in order, each budget column updated only on a strictly
      // larger value: the lowest index wins ties.
      for (int j = 0; j < n_cand[i]; ++j) {
        const int64_t w = wq[off + j];
        const double v = val[off + j];
        const double* src = prev.data();
        double* dst = cur.data();
        const uint8_t jj = static_cast<uint8_t>(j);
        for (int64_t b = w; b <= bq; ++b) {  // branch-free, so it vectorises
          const double c = src[b - w] + v;
          const bool gt = c > dst[b];
          dst[b] = gt ? c : dst[b];
          ai[b] = gt ? jj : ai[b];
        }
      }
      std::swap(prev, cur);
      off += n_cand[i];
    }
    if (!(prev[static_cast<size_t>(bq)] > ninf)) return LR_ERR_INFEASIBLE;
    // Walk back from D[n][B'].
    int64_t b = bq;
    off = total;
    for (int i = n_items - 1; i >= 0; --i) {
      off -= n_cand[i];
      const int j = arg[static_cast<size_t>(i) * width + static_cast<size_t>(b)];
      choice[i] = j;
      b -= wq[off + j];
    }
    if (objective) *objective = prev[static_cast<size_t>(bq)];
  } catch (const std::bad_alloc&) {
    return LR_ERR_NO_MEMORY;
  }
  return LR_OK;
}
