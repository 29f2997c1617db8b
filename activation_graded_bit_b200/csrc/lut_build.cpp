// Offline construction of nested look-up-table codes on the host (no GPU).
//
// Paper: Section 3.3 ("Storage Layout and Weight Loading": nested k-means codes
// satisfy the planes' nesting and need no midpoint term), Section 4 (any-precision
// LLM weights at b_max = 8, per channel) and Appendix E.2 (its k-means-based
// incremental upscaling). The library's construction, per row k of W:
//   * width 0 is one cluster holding the row; every cluster of width b - 1 is cut
//     in two at the point of its sorted members that minimises the two halves'
//     summed squared error (the optimal 1-D 2-means split), never between equal
//     values, the smallest such point on a tie; the lower half gets bit 0;
//   * a cluster with fewer than two distinct values keeps everything in its lower
//     half; an empty half takes its parent's value;
//   * entry c of width b is the mean of its members, stored as binary16 (nearest
//     even) at heap index 2^b + c of the row's 2^(b_max+1) entries (entry 0 is
//     0, entry 1 the row mean); a weight's code is its cluster at width b_max.
// Sums are compensated (Neumaier), so a cut is chosen on the criterion's value to
// within a few units in the last place of fp64.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/grinqh.h"

namespace {

// Neumaier-compensated running sum.
struct CSum {
  double s = 0.0, c = 0.0;
  void add(double v) {
    const double t = s + v;
    c += (std::fabs(s) >= std::fabs(v)) ? (s - t) + v : (v - t) + s;
    s = t;
  }
  double value() const { return s + c; }
};

// binary64 -> binary16 bits, round to nearest even, one rounding.
uint16_t to_half(double v) {
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  if (std::isnan(v)) return sign | 0x7E00;
  double a = std::fabs(v);
  if (a >= 65520.0) return sign | 0x7C00;               // rounds to infinity
  if (a < std::ldexp(1.0, -14)) {                       // subnormal range: units of 2^-24
    const double u = std::nearbyint(std::ldexp(a, 24));   // default mode: nearest even
    return sign | (uint16_t)u;                          // 1024 carries into the exponent field
  }
  int e;
  std::frexp(a, &e);                                    // a = f 2^e, f in [0.5, 1)
  const double m = std::nearbyint(std::ldexp(a, 11 - e));   // 11 significant bits
  int E = e - 1;                                        // a ~ 1.x 2^E
  uint32_t mant = (uint32_t)m;
  if (mant == 2048) { mant = 1024; ++E; }
  if (E > 15) return sign | 0x7C00;
  return sign | (uint16_t)((E + 15) << 10) | (uint16_t)(mant - 1024);
}

// Split sorted values v[lo, hi) at the best cut; returns the cut (hi when none).
int best_cut(const std::vector<double>& v, int lo, int hi) {
  const int m = hi - lo;
  if (m < 2 || !(v[lo] < v[hi - 1])) return hi;
  CSum tot;
  for (int i = lo; i < hi; ++i) tot.add(v[i]);
  const double mean = tot.value() / m;
  // S(s) = sum of the first s deviations from the mean; the between-halves sum
  // of squares S^2 m / (s (m - s)) is largest where the summed squared error is
  // smallest
  CSum dev;
  double best = -1.0;
  int cut = hi;
  for (int s = 1; s < m; ++s) {
    dev.add(v[lo + s - 1] - mean);
    if (!(v[lo + s - 1] < v[lo + s])) continue;
    const double S = dev.value();
    const double crit = S * S * (double)m / ((double)s * (double)(m - s));
    if (crit > best) {
      best = crit;
      cut = lo + s;
    }
  }
  return cut;
}

double mean_of(const std::vector<double>& v, int lo, int hi) {
  CSum t;
  for (int i = lo; i < hi; ++i) t.add(v[i]);
  return t.value() / (hi - lo);
}

}  // namespace

extern "C" grinqh_status grinqh_lut_build(const float* W, int32_t K, int32_t N, int32_t b_max, uint8_t* codes,
                                          uint16_t* lut) {
  if (!W || !codes || !lut) return GRINQH_ERR_INVALID_ARG;
  if (b_max != 2 && b_max != 4 && b_max != 6 && b_max != 8) return GRINQH_ERR_INVALID_ARG;
  if (K < 1 || N < 1 || K > (1 << 24) || N > (1 << 24)) return GRINQH_ERR_INVALID_ARG;
  for (int64_t i = 0; i < (int64_t)K * N; ++i)
    if (!std::isfinite(W[i])) return GRINQH_ERR_INVALID_ARG;
  const int E = 1 << (b_max + 1);
  std::vector<int> order(N);
  std::vector<double> v(N), cent(E);
  std::vector<int> bounds, next;   // cluster p of the current width: sorted positions [bounds[p], bounds[p+1])
  for (int32_t k = 0; k < K; ++k) {
    const float* w = W + (size_t)k * N;
    for (int n = 0; n < N; ++n) order[n] = n;
    std::sort(order.begin(), order.end(), [w](int a, int b) { return w[a] < w[b] || (w[a] == w[b] && a < b); });
    for (int i = 0; i < N; ++i) v[i] = (double)w[order[i]];
    std::fill(cent.begin(), cent.end(), 0.0);
    cent[1] = mean_of(v, 0, N);
    bounds.assign({0, N});
    for (int b = 1; b <= b_max; ++b) {
      const int np = (int)bounds.size() - 1;   // 2^(b-1) clusters
      next.assign(2 * np + 1, 0);
      for (int p = 0; p < np; ++p) {
        const int lo = bounds[p], hi = bounds[p + 1];
        const int cut = best_cut(v, lo, hi);
        next[2 * p] = lo;
        next[2 * p + 1] = cut;
        next[2 * p + 2] = hi;
        const double parent = cent[(1 << (b - 1)) + p];
        cent[(1 << b) + 2 * p] = (cut > lo) ? mean_of(v, lo, cut) : parent;
        cent[(1 << b) + 2 * p + 1] = (hi > cut) ? mean_of(v, cut, hi) : parent;
      }
      bounds.swap(next);
    }
    for (int c = 0; c < (1 << b_max); ++c)
      for (int i = bounds[c]; i < bounds[c + 1]; ++i) codes[(size_t)k * N + order[i]] = (uint8_t)c;
    uint16_t* row = lut + (size_t)k * E;
    row[0] = 0;
    for (int i = 1; i < E; ++i) row[i] = to_half(cent[i]);
  }
  return GRINQH_OK;
}
