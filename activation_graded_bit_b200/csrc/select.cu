// Per-token grading and stable per-class compaction.
//
// Paper: "GRINQH" Section 3.1 "Dynamic Precision Assignment": channel k gets the
// class j whose interval [theta_j, theta_{j+1}) holds |x_k| (theta_0 = 0,
// theta_{n+1} = inf); Section 3.2: at run time grading reduces to a few scalar
// comparisons. Here the class is the count #{ i : |x_k| >= theta_i } (ties to
// the upper class, NaN to class 0), and the channels are then listed class by
// class in ascending k, which is what the VMM kernel walks.
//
// One CTA of 1024 threads. Thread t owns the contiguous chunk
// [t*E, (t+1)*E) of channels, E = ceil(K / 1024), so "ascending thread, then
// ascending position inside the chunk" is ascending k: an exclusive scan of the
// per-thread class counts gives every channel its slot with no sorting.
#include <cstdint>
#include <cuda_fp16.h>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace grinqh {

constexpr int kSelThreads = 1024;

__device__ __forceinline__ int grade_one(uint16_t h, const float* thr, int n) {
  const float ax = fabsf(__half2float(__ushort_as_half(h)));   // exact; NaN stays NaN
  int j = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < n) j += (ax >= thr[i]) ? 1 : 0;
  return j;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t* __restrict__ x, int K,
                                                             const float* __restrict__ thresholds,
                                                             ClassTable ct, uint8_t* __restrict__ bits,
                                                             int32_t* __restrict__ idx,
                                                             int32_t* __restrict__ offsets) {
  __shared__ int s_wtot[9][32];     // per-warp class totals, then their exclusive prefix
  __shared__ float s_thr[8];
  __shared__ int s_tot[9];
  __shared__ int s_off[10];
  __shared__ uint8_t s_width[9];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = ct.n - 1;
#pragma unroll
  for (int c = 0; c < 9; ++c)
    if (tid == c && c < ct.n) s_width[c] = ct.width[c];
  pdl_wait();   // x and the thresholds may come from the kernel just before
  if (tid < n) s_thr[tid] = thresholds[tid];
  __syncthreads();
  pdl_launch_dependents();
  float thr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) thr[i] = (i < n) ? s_thr[i] : 0.0f;

  const int E = (K + kSelThreads - 1) / kSelThreads;
  const int k0 = min(K, tid * E), k1 = min(K, k0 + E);
  int cnt[9];
#pragma unroll
  for (int c = 0; c < 9; ++c) cnt[c] = 0;
  for (int k = k0; k < k1; ++k) {
    const int j = grade_one(x[k], thr, n);
#pragma unroll
    for (int c = 0; c < 9; ++c) cnt[c] += (j == c) ? 1 : 0;
    bits[k] = s_width[j];
  }

  // Block-wide exclusive scan of the nine per-thread counts: warp shuffles, then
  // one warp per class scans the 32 warp totals.
  int inc[9];
#pragma unroll
  for (int c = 0; c < 9; ++c) inc[c] = cnt[c];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int c = 0; c < 9; ++c) {
      const int v = __shfl_up_sync(0xffffffffu, inc[c], o);
      if (lane >= o) inc[c] += v;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int c = 0; c < 9; ++c) s_wtot[c][warp] = inc[c];
  }
  __syncthreads();
  if (warp < ct.n) {
    const int v = s_wtot[warp][lane];
    int w = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    s_wtot[warp][lane] = w - v;
    if (lane == 31) s_tot[warp] = w;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int c = 0; c < ct.n; ++c) { s_off[c] = acc; acc += s_tot[c]; }
    s_off[ct.n] = acc;
  }
  __syncthreads();
  if (tid <= ct.n) offsets[tid] = s_off[tid];

  int slot[9];
#pragma unroll
  for (int c = 0; c < 9; ++c) slot[c] = (c < ct.n) ? s_off[c] + s_wtot[c][warp] + inc[c] - cnt[c] : 0;
  for (int k = k0; k < k1; ++k) {
    const int j = grade_one(x[k], thr, n);
#pragma unroll
    for (int c = 0; c < 9; ++c)
      if (j == c) idx[slot[c]++] = k;
  }
}

cudaError_t launch_select(const uint16_t* x, int K, const float* thresholds, const ClassTable& ct,
                          uint8_t* bits, int32_t* idx, int32_t* offsets, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, x, K, thresholds, ct, bits, idx, offsets);
}

}  // namespace grinqh
