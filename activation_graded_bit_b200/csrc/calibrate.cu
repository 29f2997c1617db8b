// Threshold calibration by percentile mapping.
//
// Paper: "GRINQH" Section 3.2 and Appendix A.1 eq. (2): for every calibration
// sample the thresholds are the activation magnitudes that cut the sample into
// the fractions P (theta_j is the (p_0 + ... + p_{j-1})-th percentile); the
// per-sample thresholds are averaged into one static vector per layer.
//
// Order statistics come from a histogram, not a sort: binary16 magnitudes
// (sign bit cleared) order exactly like their 15-bit patterns, so one CTA per
// sample counts the 32768 possible keys in shared memory, scans the counts and
// reads off the keys at the two ranks around q_j (K-1). The interpolation
// v_lo + f * (v_hi - v_lo) and the mean over samples are done in fp64 with
// explicit round-to-nearest operations (no contraction), summing the samples in
// ascending order, then rounding once to fp32.
#include <cstdint>
#include <cuda_fp16.h>

#include "kernels.h"

namespace grinqh {

constexpr int kBins = 32768;
constexpr int kCalThreads = 1024;

__device__ __forceinline__ double key_to_f64(uint32_t key) {
  return (double)__half2float(__ushort_as_half((unsigned short)key));
}

__global__ void __launch_bounds__(kCalThreads) calib_sample_kernel(const CalibArgs a) {
  extern __shared__ uint32_t hist[];      // kBins counters
  __shared__ uint32_t s_wsum[32];
  __shared__ uint32_t s_key[16];
  const int s = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  for (int b = tid; b < kBins; b += kCalThreads) hist[b] = 0u;
  __syncthreads();
  const uint16_t* xs = a.X + (size_t)s * a.K;
  for (int k = tid; k < a.K; k += kCalThreads) atomicAdd(&hist[xs[k] & 0x7FFFu], 1u);
  __syncthreads();

  // thread t owns bins [32t, 32t+32): block exclusive scan of the chunk totals
  const int base = tid * 32;
  uint32_t local = 0;
#pragma unroll 8
  for (int e = 0; e < 32; ++e) local += hist[base + ((e + lane) & 31)];
  uint32_t inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) s_wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = s_wsum[lane];
    uint32_t w = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    s_wsum[lane] = w - v;
  }
  __syncthreads();
  const uint32_t excl = s_wsum[warp] + inc - local;

  // locate the keys at ranks lo_j and hi_j
  for (int q = 0; q < 2 * a.n; ++q) {
    if (a.mode[q >> 1] != 0) continue;
    const uint32_t rank = (uint32_t)((q & 1) ? a.hi[q >> 1] : a.lo[q >> 1]);
    if (rank >= excl && rank < excl + local) {
      uint32_t cum = excl;
      for (int e = 0; e < 32; ++e) {
        const uint32_t h = hist[base + e];
        if (rank < cum + h) { s_key[q] = (uint32_t)(base + e); break; }
        cum += h;
      }
    }
  }
  __syncthreads();
  if (tid < a.n && a.mode[tid] == 0) {
    const double vlo = key_to_f64(s_key[2 * tid]);
    const double vhi = key_to_f64(s_key[2 * tid + 1]);
    const double th = __dadd_rn(vlo, __dmul_rn(a.frac[tid], __dsub_rn(vhi, vlo)));
    a.per_sample[(size_t)s * a.n + tid] = th;
  }
}

__global__ void calib_mean_kernel(const CalibArgs a) {
  const int j = threadIdx.x;
  if (j >= a.n) return;
  float out;
  if (a.mode[j] == 2) {
    out = __int_as_float(0x7f800000);
  } else if (a.mode[j] == 1) {
    out = 0.0f;
  } else {
    double sum = 0.0;
    for (int s = 0; s < a.S; ++s) sum = __dadd_rn(sum, a.per_sample[(size_t)s * a.n + j]);
    out = __double2float_rn(__ddiv_rn(sum, (double)a.S));
  }
  a.thresholds[j] = out;
}

size_t calibrate_workspace_bytes(int S, int n) {
  return ((size_t)S * (n > 0 ? n : 1) * sizeof(double) + 15) & ~(size_t)15;
}

cudaError_t launch_calibrate(const CalibArgs& a, cudaStream_t st) {
  if (a.n <= 0) return cudaSuccess;
  const int smem = kBins * (int)sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(calib_sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  calib_sample_kernel<<<a.S, kCalThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  calib_mean_kernel<<<1, 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace grinqh
