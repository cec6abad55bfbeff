// KV-COBRA rank/bit allocation (calibration-time host code).
//
// KV-COBRA explainer, section "The news": per head, step C1 chooses the rank r
// (directions kept) and bit width b where dropping directions -- whose variance
// is lost outright -- and the rounding noise of the kept directions balance;
// step C2 moves budget across heads until no extra bit anywhere removes more
// error than it costs ("water-filling").  The error model of one head is
//   E(r, b) = sum_{i >= r} lambda_i + eps_b * sum_{i < r} lambda_i
// with lambda the head's direction variances in decreasing order and eps_b the
// relative rounding noise of the b-bit quantizer (measured by the caller).
// C2 starts every head at (16, 1) and repeatedly applies the single affordable
// upgrade with the largest error reduction per extra bit (ties: lower head,
// then fewer bits) until none fits or none helps.
#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/kvq.h"

namespace {

constexpr int kRanks[5] = {16, 32, 64, 96, 128};

double head_error(const double* lambda, int r, int b, const double* eps) {
  double kept = 0.0, lost = 0.0;
  for (int i = 0; i < KVQ_HEAD_DIM; ++i) {
    if (i < r) kept += lambda[i];
    else lost += lambda[i];
  }
  return lost + eps[b - 1] * kept;
}

}  // namespace

extern "C" kvq_status kvq_cobra_allocate(int n_heads, const double* lambdas, double bpd, const double* eps,
                                         int* ranks, int* bits, int* bits_used) {
  if (n_heads < 1 || !lambdas || !eps || !ranks || !bits) return KVQ_ERR_INVALID_ARG;
  if (!(bpd > 0.0) || !std::isfinite(bpd)) return KVQ_ERR_INVALID_ARG;
  for (int h = 0; h < n_heads; ++h)
    for (int i = 0; i < KVQ_HEAD_DIM; ++i) {
      const double v = lambdas[(size_t)h * KVQ_HEAD_DIM + i];
      if (!(v >= 0.0) || !std::isfinite(v)) return KVQ_ERR_INVALID_ARG;
      if (i > 0 && v > lambdas[(size_t)h * KVQ_HEAD_DIM + i - 1]) return KVQ_ERR_INVALID_ARG;  // must be sorted
    }
  const int budget = (int)(bpd * KVQ_HEAD_DIM * n_heads + 0.5);
  if (budget < 16 * n_heads) return KVQ_ERR_CAPACITY;
  // the 20 candidate errors of every head, computed once
  std::vector<double> err((size_t)n_heads * 20);
  for (int h = 0; h < n_heads; ++h)
    for (int ri = 0; ri < 5; ++ri)
      for (int b = 1; b <= 4; ++b)
        err[(size_t)h * 20 + ri * 4 + (b - 1)] = head_error(lambdas + (size_t)h * KVQ_HEAD_DIM, kRanks[ri], b, eps);
  int used = 0;
  for (int h = 0; h < n_heads; ++h) { ranks[h] = 16; bits[h] = 1; used += 16; }
  std::vector<double> cur_err(n_heads);
  for (int h = 0; h < n_heads; ++h) cur_err[h] = err[(size_t)h * 20];
  for (;;) {
    int best_h = -1, best_r = 0, best_b = 0, best_bits = 0;
    double best_gain = 0.0, best_err = 0.0;
    for (int h = 0; h < n_heads; ++h) {
      const int cur = ranks[h] * bits[h];
      for (int ri = 0; ri < 5; ++ri)
        for (int b = 1; b <= 4; ++b) {
          const int nb = kRanks[ri] * b;
          if (nb <= cur || used - cur + nb > budget) continue;
          const double e = err[(size_t)h * 20 + ri * 4 + (b - 1)];
          const double gain = (cur_err[h] - e) / (double)(nb - cur);
          if (gain > best_gain || (gain == best_gain && gain > 0.0 && best_h == h && nb < best_bits)) {
            best_gain = gain; best_h = h; best_r = kRanks[ri]; best_b = b; best_bits = nb; best_err = e;
          }
        }
    }
    if (best_h < 0) break;
    used += best_bits - ranks[best_h] * bits[best_h];
    ranks[best_h] = best_r;
    bits[best_h] = best_b;
    cur_err[best_h] = best_err;
  }
  if (bits_used) *bits_used = used;
  return KVQ_OK;
}
