// Verify-length scheduler (host logic, no device work).
//
// mkdocs.reaper.mx DeepSeek-V4.1-Flash "06-extensions", DSpark table: the
// scheduler picks each request's verify length from the confidence head's
// prefix survival probabilities and throughput curves of the engine measured
// beforehand, maximising the expected system throughput at the current load.
// aigest.pl "DeepSeek prezentuje DSpark", "Optymalizacja weryfikacji i
// wydajności": the curve is SPS(B), profiled once at start-up; idle GPUs
// verify more tokens, busy ones fewer; the early-stopping rule keeps the
// method lossless (rejection sampling still verifies every kept position).
//
// Objective, for verify lengths k_b in 1..K:
//   S_{b,i} = prod_{j<=i} clamp(c_{b,j}, 0, 1)            (NaN score -> 0)
//   E(k)    = sum_b (1 + sum_{i<k_b} S_{b,i})             expected tokens per step
//   T(k)    = E(k) * SPS(sum_b (k_b + 1))                 tokens per second
// Each request costs k_b + 1 target rows (its drafts and the bonus row).
//
// For a fixed total m = sum k_b the largest E takes, on top of k_b = 1, the
// m - B largest survivals S_{b,i} with i >= 1.  S is non-increasing along a
// row (every factor is in [0,1], and a rounded product of a representable
// value and a factor <= 1 never exceeds that value), so sorting all S_{b,i}
// in descending order, ties by (b, i) ascending, gives a list whose every
// prefix is a valid allocation: position i of a row comes after position
// i - 1.  One pass over that list evaluates T at every total and keeps the
// first (smallest-total) maximum.  O(BK log BK).
#include "specdec.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

namespace {

struct Gain {
  double s;
  int32_t b;
  int32_t i;
};

}  // namespace

extern "C" spec_status spec_schedule_verify_len(const float *conf, int32_t B, int32_t K,
                                                const double *sps, int32_t n_sps,
                                                int32_t *verify_len, double *expected) {
  if (!conf || !sps || !verify_len || B < 1 || K < 1 || n_sps < 1 ||
      (int64_t)B * K > (int64_t{1} << 26))
    return SPEC_ERR_INVALID_ARG;
  for (int32_t m = 0; m < n_sps; ++m)
    if (!std::isfinite(sps[m]) || sps[m] < 0.0) return SPEC_ERR_INVALID_ARG;

  std::vector<Gain> gains;
  gains.reserve((size_t)B * (size_t)(K - 1));
  double e = 0.0;  // expected tokens with every k_b = 1
  for (int32_t b = 0; b < B; ++b) {
    double s = 1.0;
    for (int32_t i = 0; i < K; ++i) {
      float c = conf[(size_t)b * K + i];
      double f = std::isnan(c) ? 0.0 : std::min(1.0, std::max(0.0, (double)c));
      s *= f;
      if (i == 0)
        e += 1.0 + s;
      else
        gains.push_back({s, b, i});
    }
  }
  std::sort(gains.begin(), gains.end(), [](const Gain &x, const Gain &y) {
    if (x.s != y.s) return x.s > y.s;
    if (x.b != y.b) return x.b < y.b;
    return x.i < y.i;
  });

  auto rate = [&](int64_t m) { return m < n_sps ? sps[m] : 0.0; };
  const int64_t m0 = 2 * (int64_t)B;  // target rows with every k_b = 1
  double best_t = e * rate(m0), best_e = e;
  size_t take = 0;
  for (size_t j = 0; j < gains.size(); ++j) {
    e += gains[j].s;
    double t = e * rate(m0 + (int64_t)j + 1);
    if (t > best_t) {
      best_t = t;
      best_e = e;
      take = j + 1;
    }
  }
  for (int32_t b = 0; b < B; ++b) verify_len[b] = 1;
  for (size_t j = 0; j < take; ++j)
    verify_len[gains[j].b] = std::max(verify_len[gains[j].b], gains[j].i + 1);
  if (expected) {
    expected[0] = best_e;
    expected[1] = best_t;
  }
  return SPEC_OK;
}
