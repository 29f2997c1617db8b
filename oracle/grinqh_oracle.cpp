// GRINQH reference oracle: plain, slow, fp64 CPU implementation.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
// this file. Only the test suite, the package smoke check and the benchmark's
// CPU-baseline leg use it. It shares no code with the CUDA library: every
// definition below is written out again from the paper
//   "GRINQH: Graded Input-based Quantization Hierarchy for Efficient LLM
//    Generation" (arXiv 2606.23419)
// and from the library conventions stated next to each function.
//
// Conventions (shared by the paper's text and this library's contract):
//   W is K x N (K input channels = rows, N output channels = columns), stored
//   input-major as in Section 3.3 "Storage Layout and Weight Loading" and
//   Appendix C.1 "Sparse bit-loading". Groups are 128 consecutive columns of one
//   row (G = 128, Section 4 "Models and Baselines"). fp16 values travel as IEEE
//   binary16 bit patterns in uint16_t.
//
// Parity status: every function here is pinned by a CPU test against a closed
// form, an invariant, a library routine or brute force (tests/test_oracle_*.py).
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---------------------------------------------------------------------------
// IEEE 754 binary16 <-> binary64, written from the format definition:
// 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; exponent field 0 is
// zero/subnormal (value f * 2^-24), field 31 is infinity/NaN.
// ---------------------------------------------------------------------------
double orc_f16_to_f64(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  double v;
  if (e == 0) {
    v = std::ldexp((double)f, -24);
  } else if (e == 31) {
    v = (f == 0) ? INFINITY : NAN;
  } else {
    v = std::ldexp((double)(1024 + f), e - 25);
  }
  return sign ? -v : v;
}

// Round-to-nearest-even conversion straight from binary64 (no detour through
// binary32, which would round twice).
uint16_t orc_f64_to_f16(double v) {
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  if (std::isnan(v)) return sign | 0x7E00;
  const double a = std::fabs(v);
  // The largest finite half is 65504 = 2047 * 2^5; the halfway point to the
  // next power of two (65536) is 65520, and the tie goes to the even
  // significand 2048, i.e. to infinity.
  if (a >= 65520.0) return sign | 0x7C00;
  if (a < std::ldexp(1.0, -14)) {
    // subnormal range: value = m * 2^-24, m in [0, 1024]; m = 1024 encodes the
    // smallest normal number, which is what the bit pattern 0x0400 means.
    const double m = std::nearbyint(std::ldexp(a, 24));
    return sign | (uint16_t)m;
  }
  int e2;
  std::frexp(a, &e2);              // a = f * 2^e2 with f in [0.5, 1)
  int E = e2 - 1;                  // a in [2^E, 2^(E+1))
  double m = std::nearbyint(std::ldexp(a, 10 - E));   // significand in [1024, 2048]
  if (m == 2048.0) { m = 1024.0; E += 1; }
  return sign | (uint16_t)((E + 15) << 10) | (uint16_t)(m - 1024.0);
}

// ---------------------------------------------------------------------------
// RTN asymmetric quantisation to b_max bits per (row k, 128-column group g).
// Paper: Section 3.3 (every weight w_ij becomes one b_max-bit integer whose
// scale s and zero point z are set once at the full b_max precision; the
// evaluation uses b_max in {4, 6, 8}), Section 4 (RTN, G = 128) and Appendix E.1 (the RTN
// model at b_max is the parent of every truncated width).
// Library convention, with L = 2^b_max - 1 levels: s = fp16(range / L) rounded
// to nearest even straight from fp64, s := 1 if that rounds to 0, s := 65504
// if it overflows; z = clamp(rne(-min / s), 0, L) stored as fp16 (exact, and +0
// rather than -0); q = clamp(rne(w / s) + z, 0, L). Quotients are taken in
// fp64; for a binary32 numerator and a binary16 denominator the fp64 quotient
// never lands on, or crosses, a half-integer that the exact quotient does not,
// so rne of it equals rne of the exact rational.
// Outputs: q[K*N] row-major, scale[K*n_g], zero[K*n_g] with n_g = ceil(N/128).
// Returns 0, or -1 on bad sizes or b_max outside 1..8.
// ---------------------------------------------------------------------------
int orc_rtn_quantize_bmax(const float* W, int K, int N, int bmax, uint8_t* q, uint16_t* scale,
                          uint16_t* zero) {
  if (K <= 0 || N <= 0 || bmax < 1 || bmax > 8) return -1;
  const double levels = (double)((1 << bmax) - 1);
  const int ng = (N + 127) / 128;
  for (int k = 0; k < K; ++k) {
    for (int g = 0; g < ng; ++g) {
      const int c0 = g * 128, c1 = std::min(N, c0 + 128);
      double mn = INFINITY, mx = -INFINITY;
      for (int n = c0; n < c1; ++n) {
        const double w = (double)W[(size_t)k * N + n];
        if (w < mn) mn = w;
        if (w > mx) mx = w;
      }
      const double range = mx - mn;
      uint16_t sb = orc_f64_to_f16(range / levels);
      double s = orc_f16_to_f64(sb);
      if (s == 0.0) { sb = 0x3C00; s = 1.0; }
      if (std::isinf(s)) { sb = 0x7BFF; s = 65504.0; }
      double z = std::nearbyint(-mn / s);
      if (z < 0.0) z = 0.0;
      if (z > levels) z = levels;
      z = z + 0.0;   // a zero point of -0 (min = +0) is stored as +0
      scale[(size_t)k * ng + g] = sb;
      zero[(size_t)k * ng + g] = orc_f64_to_f16(z);
      for (int n = c0; n < c1; ++n) {
        double v = std::nearbyint((double)W[(size_t)k * N + n] / s) + z;
        if (v < 0.0) v = 0.0;
        if (v > levels) v = levels;
        q[(size_t)k * N + n] = (uint8_t)v;
      }
    }
  }
  return 0;
}

// The 8-bit case (b_max = 8, 255 levels), the library's default layout.
int orc_rtn_quantize(const float* W, int K, int N, uint8_t* q, uint16_t* scale, uint16_t* zero) {
  return orc_rtn_quantize_bmax(W, K, N, 8, q, scale, zero);
}

// ---------------------------------------------------------------------------
// Nested reconstruction code of a b_max-bit code q read at width b.
// Paper: Section 3.3, "Weight Reconstruction and Bias Correction": the top b
// bits q_b, scaled back by 2^(b_max - b), plus the midpoint term
// phi = 2^(b_max - b - 1). Library convention: phi is applied for
// 1 <= b < b_max only (b = b_max reads q unchanged); b = 0 means the row is
// skipped entirely, and these functions return -1 for it.
// ---------------------------------------------------------------------------
int orc_code_bmax(int q, int b, int bmax) {
  if (b <= 0) return -1;
  if (b >= bmax) return q;
  const int qb = q >> (bmax - b);         // the b most significant of the b_max bits
  return qb * (1 << (bmax - b)) + (1 << (bmax - b - 1));
}

int orc_code(int q, int b) { return orc_code_bmax(q, b, 8); }

// ---------------------------------------------------------------------------
// Full-width dequantisation for the prefill product.
// Paper: Section 4 ("Prefill vs. Decoding Evaluation": prefill unpacks the
// weights at full b_max precision and runs a dense matrix-matrix product) and
// Section 3.3 (w_hat = s * (q - z) at b = b_max). Library reading: the dense
// operand is w_hat rounded once to binary16 (round to nearest even), computed
// as the exact fp64 product s * (q - z) (an 11-bit by 9-bit product).
// q[K*N] codes of b_max bits, scale/zero [K*n_g] fp16 bit patterns; out[K*N]
// binary16 bit patterns. Returns 0, or -1 on bad sizes.
// ---------------------------------------------------------------------------
int orc_dequant_f16(const uint8_t* q, const uint16_t* scale, const uint16_t* zero, int K, int N,
                    uint16_t* out) {
  if (K <= 0 || N <= 0) return -1;
  const int ng = (N + 127) / 128;
  for (int k = 0; k < K; ++k)
    for (int n = 0; n < N; ++n) {
      const double s = orc_f16_to_f64(scale[(size_t)k * ng + n / 128]);
      const double z = orc_f16_to_f64(zero[(size_t)k * ng + n / 128]);
      out[(size_t)k * N + n] = orc_f64_to_f16(s * ((double)q[(size_t)k * N + n] - z));
    }
  return 0;
}

// ---------------------------------------------------------------------------
// Grading. Paper: Section 3.1 "Dynamic Precision Assignment": b_i = b_k when
// |x_i| lies in [theta_k, theta_{k+1}) with theta_0 = 0 and theta_{n+1} = inf.
// Written as a count: class j = #{ i in 1..n : |x| >= theta_i }, which equals
// the interval rule for non-decreasing thresholds and is defined for any.
// NaN magnitudes compare false everywhere and land in class 0.
// x: K fp16 bit patterns; theta: n fp32 values; classes: n+1 bit widths.
// Output bits[k] = classes[j_k].
// ---------------------------------------------------------------------------
int orc_grade(const uint16_t* x, int K, const float* theta, int n_theta,
              const uint8_t* classes, uint8_t* bits) {
  if (K < 0 || n_theta < 0 || n_theta > 8) return -1;
  for (int k = 0; k < K; ++k) {
    const double ax = std::fabs(orc_f16_to_f64(x[k]));
    int j = 0;
    for (int i = 0; i < n_theta; ++i)
      if (ax >= (double)theta[i]) ++j;
    bits[k] = classes[j];
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Stable compaction of channel indices per class: class-major, ascending k
// inside each class. offsets[j] = number of channels in classes below j, and
// offsets[n_classes] = K. (The paper's kernel "loads the b/2 most significant
// segments" per row, Section 3.3; the per-class index lists are this library's
// way of handing that row set to the kernel.)
// ---------------------------------------------------------------------------
int orc_compact(const uint8_t* bits, int K, const uint8_t* classes, int n_classes,
                int32_t* idx, int32_t* offsets) {
  if (K < 0 || n_classes < 1 || n_classes > 9) return -1;
  int pos = 0;
  for (int j = 0; j < n_classes; ++j) {
    offsets[j] = pos;
    for (int k = 0; k < K; ++k)
      if (bits[k] == classes[j]) idx[pos++] = k;
  }
  offsets[n_classes] = pos;
  return pos == K ? 0 : -2;   // -2: some bit width is not in the class set
}

// ---------------------------------------------------------------------------
// The graded vector-matrix product, in fp64.
// Paper: Section 3 / Fig. 2 (only the top b_k bits of row k take part, b = 0
// rows are bypassed) and the reconstruction of Section 3.3 with the library's
// zero-point form w_hat = s * (code - z), code = orc_code_bmax(q, b, b_max).
// y[n] = sum over k ascending with bits[k] > 0 of x_k * w_hat[k][n];
// bound[n] = sum of |x_k * w_hat[k][n]| over the same k (the scale of the
// parity tolerance). x, scale, zero are fp16 bit patterns.
// nthreads > 1 splits the COLUMNS across OpenMP threads; every y[n] is still
// summed over k in ascending order.
// ---------------------------------------------------------------------------
int orc_vmm_bmax(const uint16_t* x, const uint8_t* q, const uint16_t* scale, const uint16_t* zero,
                 const uint8_t* bits, int K, int N, int bmax, double* y, double* bound, int nthreads) {
  if (K < 0 || N <= 0 || bmax < 1 || bmax > 8) return -1;
  const int ng = (N + 127) / 128;
  for (int n = 0; n < N; ++n) { y[n] = 0.0; if (bound) bound[n] = 0.0; }
  if (nthreads < 1) nthreads = 1;
  const int nchunks = nthreads;
#pragma omp parallel for num_threads(nthreads) schedule(static, 1) if (nthreads > 1)
  for (int t = 0; t < nchunks; ++t) {
    const int n0 = (int)((long long)N * t / nchunks);
    const int n1 = (int)((long long)N * (t + 1) / nchunks);
    for (int k = 0; k < K; ++k) {
      const int b = bits[k];
      if (b == 0) continue;
      const double xk = orc_f16_to_f64(x[k]);
      for (int n = n0; n < n1; ++n) {
        const int g = n / 128;
        const double s = orc_f16_to_f64(scale[(size_t)k * ng + g]);
        const double z = orc_f16_to_f64(zero[(size_t)k * ng + g]);
        const double w = s * ((double)orc_code_bmax(q[(size_t)k * N + n], b, bmax) - z);
        const double t2 = xk * w;
        y[n] += t2;
        if (bound) bound[n] += std::fabs(t2);
      }
    }
  }
  return 0;
}

int orc_vmm(const uint16_t* x, const uint8_t* q, const uint16_t* scale, const uint16_t* zero,
            const uint8_t* bits, int K, int N, double* y, double* bound, int nthreads) {
  return orc_vmm_bmax(x, q, scale, zero, bits, K, N, 8, y, bound, nthreads);
}

// ---------------------------------------------------------------------------
// Maximum-entropy precision distribution for a requested average width.
// Paper: Appendix A.1, eq. (1) constrains P to the simplex with
// |sum_i p_i b_i - b*| <= eps and leaves the objective to a model metric that
// needs trained models. Library reading: among all P meeting the constraint
// exactly, take the one of maximum entropy, p_i proportional to
// exp(lambda * b_i), with lambda found by bisection in fp64 (the mean width is
// increasing in lambda). b* = b_0 or b* = b_n give the one-hot end classes;
// b* outside [b_0, b_n] is an error (-1).
// ---------------------------------------------------------------------------
static void orc_gibbs(const uint8_t* b, int m, double lam, double* p) {
  // shift the exponent by the end class on the side lam points to, so that
  // every exponential is at most 1
  const double c = lam >= 0.0 ? (double)b[m - 1] : (double)b[0];
  double z = 0.0;
  for (int i = 0; i < m; ++i) { p[i] = std::exp(lam * ((double)b[i] - c)); z += p[i]; }
  for (int i = 0; i < m; ++i) p[i] /= z;
}

static double orc_mean_bits(const uint8_t* b, int m, const double* p) {
  double s = 0.0;
  for (int i = 0; i < m; ++i) s += p[i] * (double)b[i];
  return s;
}

int orc_maxent_distribution(const uint8_t* classes, int n_classes, double target, double* P) {
  if (n_classes < 1 || n_classes > 9) return -1;
  for (int i = 1; i < n_classes; ++i) if (classes[i] <= classes[i - 1]) return -1;
  const double lo_b = classes[0], hi_b = classes[n_classes - 1];
  if (!(target >= lo_b && target <= hi_b)) return -1;
  for (int i = 0; i < n_classes; ++i) P[i] = 0.0;
  if (target == hi_b) { P[n_classes - 1] = 1.0; return 0; }
  if (target == lo_b) { P[0] = 1.0; return 0; }
  std::vector<double> p(n_classes);
  double L = 1.0;
  for (int it = 0; it < 64; ++it) {
    orc_gibbs(classes, n_classes, L, p.data());
    const double up = orc_mean_bits(classes, n_classes, p.data());
    orc_gibbs(classes, n_classes, -L, p.data());
    const double dn = orc_mean_bits(classes, n_classes, p.data());
    if (up > target && dn < target) break;
    L *= 2.0;
  }
  double a = -L, c = L;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (a + c);
    if (mid == a || mid == c) break;
    orc_gibbs(classes, n_classes, mid, p.data());
    if (orc_mean_bits(classes, n_classes, p.data()) < target) a = mid; else c = mid;
  }
  orc_gibbs(classes, n_classes, 0.5 * (a + c), P);
  return 0;
}

// ---------------------------------------------------------------------------
// Threshold calibration by percentile mapping.
// Paper: Section 3.2: theta_k is the (sum_{j<k} p_j)-th percentile of the
// activation magnitudes of each calibration sample, and the per-sample values
// are averaged into one static threshold vector; Appendix A.1 eq. (2).
// Library readings: n thresholds for n+1 classes; percentile = linear
// interpolation at position q*(K-1) of the ascending magnitudes; mean over the
// S samples summed in ascending sample order in fp64, then rounded to fp32.
// theta_j = 0 when q_j is exactly 0; theta_j = +inf when every class from j on
// has p = 0 (those classes are never selected).
// X: S rows of K fp16 bit patterns. P: n_classes probabilities (each >= 0,
// summing to 1 within 1e-9). theta: n_classes - 1 outputs. Returns 0 or -1.
// ---------------------------------------------------------------------------
int orc_thresholds(const uint16_t* X, int S, int K, const double* P, int n_classes, float* theta) {
  if (S < 1 || K < 1 || n_classes < 1 || n_classes > 9) return -1;
  double tot = 0.0;
  for (int i = 0; i < n_classes; ++i) { if (!(P[i] >= 0.0)) return -1; tot += P[i]; }
  if (std::fabs(tot - 1.0) > 1e-9) return -1;
  const int n = n_classes - 1;
  std::vector<double> qj(n + 1, 0.0);
  {
    double acc = 0.0;
    for (int j = 1; j <= n; ++j) { acc += P[j - 1]; qj[j] = acc; }
  }
  std::vector<double> sum(n + 1, 0.0);
  std::vector<double> v(K);
  for (int s = 0; s < S; ++s) {
    for (int k = 0; k < K; ++k) v[k] = std::fabs(orc_f16_to_f64(X[(size_t)s * K + k]));
    std::sort(v.begin(), v.end());
    for (int j = 1; j <= n; ++j) {
      const double pos = qj[j] * (double)(K - 1);
      double th;
      if (pos >= (double)(K - 1)) {
        th = v[K - 1];
      } else {
        const double fl = std::floor(pos);
        const int lo = (int)fl;
        const int hi = std::min(lo + 1, K - 1);
        const double fr = pos - fl;
        th = v[lo] + fr * (v[hi] - v[lo]);
      }
      sum[j] += th;
    }
  }
  for (int j = 1; j <= n; ++j) {
    bool tail_empty = true;
    for (int i = j; i < n_classes; ++i) if (P[i] != 0.0) tail_empty = false;
    if (tail_empty) theta[j - 1] = INFINITY;
    else if (qj[j] == 0.0) theta[j - 1] = 0.0f;
    else theta[j - 1] = (float)(sum[j] / (double)S);
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Nested non-uniform (look-up table) codes.
// Paper: Section 3.3 "Storage Layout and Weight Loading": the bit planes need a
// nested quantisation, which uniform codes and k-means codes such as
// any-precision LLM's satisfy; for non-uniform weights the parent model has
// b_max bits, and the midpoint term is not used because the nested levels are
// already centred. Section 4 "Models and Baselines": any-precision LLM weights
// at b_max = 8, per channel. Appendix E.2: the same framework on nested
// any-precision weights, built by k-means-based incremental upscaling.
//
// Library reading (the pages give no construction of their own):
//  * one table per row k (the axis the planes are graded on) and width b: the
//    code c_b = q >> (b_max - b) (the top b bits of the b_max-bit code, as for
//    uniform codes) selects the level-b centroid of the row; w_hat = that value.
//  * tables in heap order: entry 2^b + c is centroid c of width b, so width b
//    occupies entries [2^b, 2^(b+1)) of the row's 2^(b_max+1) entries (entry 1
//    is the row mean, entry 0 is unused and 0), stored as binary16 (RNE).
//  * incremental upscaling: width 0 is one cluster holding the whole row; each
//    cluster of width b-1 is split in two by the optimal one-dimensional
//    2-means split of its members (lower child bit 0, upper child bit 1). On
//    sorted values an optimal split is a cut between two neighbours; a cut
//    between equal values is not used, so equal weights share a code. The cut
//    maximises the between-cluster sum of squares S^2 m / (s (m - s)) (S the sum
//    of the s lower members' deviations from the cluster mean, m members), which
//    is the same as minimising the two children's summed squared error; ties go
//    to the smallest s. A cluster with fewer than two distinct values keeps all
//    members in its lower child; an empty child's centroid is its parent's.
//  * centroids are the fp64 means of their members (each child of a split then
//    averages, weighted by its count, to its parent).
// W fp32 [K*N] row-major; q out [K*N] codes of bmax bits; lut out [K*2^(bmax+1)]
// binary16 bit patterns; cent (optional) [K*2^(bmax+1)] the same centroids in
// fp64. Returns 0, or -1 on bad sizes.
// ---------------------------------------------------------------------------
int orc_lut_build(const float* W, int K, int N, int bmax, uint8_t* q, uint16_t* lut, double* cent) {
  if (K <= 0 || N <= 0 || bmax < 1 || bmax > 8) return -1;
  const int E = 1 << (bmax + 1);
  std::vector<double> c(E);
  std::vector<int> order(N), code(N);
  for (int k = 0; k < K; ++k) {
    const float* w = W + (size_t)k * N;
    for (int n = 0; n < N; ++n) order[n] = n;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return w[a] < w[b]; });
    std::fill(c.begin(), c.end(), 0.0);
    std::fill(code.begin(), code.end(), 0);
    // members of each cluster are a contiguous run of `order`: run [lo, hi)
    std::vector<int> lo(1, 0), hi(1, N);
    double root = 0.0;
    for (int n = 0; n < N; ++n) root += (double)w[n];
    c[1] = root / (double)N;
    for (int b = 1; b <= bmax; ++b) {
      std::vector<int> nlo(2 * lo.size()), nhi(2 * lo.size());
      for (size_t p = 0; p < lo.size(); ++p) {
        const int a = lo[p], e = hi[p], m = e - a;
        const double parent = c[(1 << (b - 1)) + (int)p];
        int cut = e;   // lower child [a, cut), upper child [cut, e)
        if (m >= 2) {
          double mean = 0.0;
          for (int i = a; i < e; ++i) mean += (double)w[order[i]];
          mean /= (double)m;
          double S = 0.0, best = -1.0;
          for (int s = 1; s < m; ++s) {
            S += (double)w[order[a + s - 1]] - mean;
            if (!(w[order[a + s - 1]] < w[order[a + s]])) continue;   // no cut between equal values
            const double B = S * S * (double)m / ((double)s * (double)(m - s));
            if (B > best) { best = B; cut = a + s; }
          }
        }
        nlo[2 * p] = a; nhi[2 * p] = cut;
        nlo[2 * p + 1] = cut; nhi[2 * p + 1] = e;
        for (int ch = 0; ch < 2; ++ch) {
          const int ca = nlo[2 * p + ch], ce = nhi[2 * p + ch];
          double v = parent;
          if (ce > ca) {
            double t = 0.0;
            for (int i = ca; i < ce; ++i) t += (double)w[order[i]];
            v = t / (double)(ce - ca);
          }
          c[(1 << b) + 2 * (int)p + ch] = v;
          for (int i = ca; i < ce; ++i) code[order[i]] = 2 * (int)p + ch;
        }
      }
      lo.swap(nlo);
      hi.swap(nhi);
    }
    for (int n = 0; n < N; ++n) q[(size_t)k * N + n] = (uint8_t)code[n];
    for (int i = 0; i < E; ++i) {
      lut[(size_t)k * E + i] = (i == 0) ? 0 : orc_f64_to_f16(c[i]);
      if (cent) cent[(size_t)k * E + i] = (i == 0) ? 0.0 : c[i];
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Graded product over nested table codes (the reading above): for b_k > 0,
// w_hat[k][n] = lut[k][2^b_k + (q[k][n] >> (bmax - b_k))] (binary16), no
// midpoint, no scale or zero point; y[n] = sum over k ascending of
// x_k * w_hat[k][n], bound[n] = sum of |x_k * w_hat[k][n]|. A width above
// bmax is an error. nthreads > 1 splits the columns as orc_vmm_bmax does.
// ---------------------------------------------------------------------------
int orc_vmm_lut(const uint16_t* x, const uint8_t* q, const uint16_t* lut, const uint8_t* bits, int K, int N,
                int bmax, double* y, double* bound, int nthreads) {
  if (K < 0 || N <= 0 || bmax < 1 || bmax > 8) return -1;
  for (int k = 0; k < K; ++k) if (bits[k] > bmax) return -1;
  const int E = 1 << (bmax + 1);
  for (int n = 0; n < N; ++n) { y[n] = 0.0; if (bound) bound[n] = 0.0; }
  if (nthreads < 1) nthreads = 1;
  const int nchunks = nthreads;
#pragma omp parallel for num_threads(nthreads) schedule(static, 1) if (nthreads > 1)
  for (int t = 0; t < nchunks; ++t) {
    const int n0 = (int)((long long)N * t / nchunks);
    const int n1 = (int)((long long)N * (t + 1) / nchunks);
    for (int k = 0; k < K; ++k) {
      const int b = bits[k];
      if (b == 0) continue;
      const double xk = orc_f16_to_f64(x[k]);
      const uint16_t* row = lut + (size_t)k * E + (1 << b);
      for (int n = n0; n < n1; ++n) {
        const double w = orc_f16_to_f64(row[q[(size_t)k * N + n] >> (bmax - b)]);
        const double t2 = xk * w;
        y[n] += t2;
        if (bound) bound[n] += std::fabs(t2);
      }
    }
  }
  return 0;
}

}  // extern "C"
