// Per-token grading and stable per-class compaction.
//
// Paper: "GRINQH" Section 3.1 "Dynamic Precision Assignment": channel k gets the
// class j whose interval [theta_j, theta_{j+1}) holds |x_k| (theta_0 = 0,
// theta_{n+1} = inf); Section 3.2: at run time grading reduces to a few scalar
// comparisons. Here the class is the count #{ i : |x_k| >= theta_i } (ties to
// the upper class, NaN to class 0), and the channels are then listed class by
// class in ascending k, which is what the VMM kernel walks.
//
// One CTA of 512 threads per chunk of 1024 channels, with no communication
// between CTAs:
//  * every CTA streams all of x once (a few KB, resident in L2; its loads go out
//    together with the chunk's own, so the CTA waits for one memory round trip)
//    and counts, for each threshold, the channels whose |x| reaches it, both
//    over the whole vector and over the channels before its own chunk (a
//    snapshot of the running counts taken where the stream crosses the chunk
//    start). The count compares two channels per fp16 instruction and keeps
//    per-warp totals in shared memory (no atomics). Ordered by their overall
//    count, the thresholds are in ascending order, so no sort of the thresholds
//    is needed: the counts at sorted position c give the number of channels of
//    class > c overall and before the chunk, hence the class offsets and this
//    chunk's first slot in each class;
//  * inside the chunk, round e of thread t grades channel lo + 512 e + t, so
//    (round, warp, lane) order is ascending k; one ballot per class and round gives
//    each channel its rank among the warp's channels of that class, and one warp
//    per class scans the 32 (round, warp) counts.
// The class count does not depend on the order of the thresholds, so grading
// against them as given yields the j of the definition.
#include <cstdint>
#include <cuda_fp16.h>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace grinqh {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelChunk = 1024;
constexpr int kSelRounds = kSelChunk / kSelThreads;   // 2
constexpr int kNoClass = 15;

static_assert(kSelRounds * kSelWarps == 32, "one scan lane per (round, warp)");

__device__ __forceinline__ float abs_half(uint16_t h) {
  return __half2float(__ushort_as_half((uint16_t)(h & 0x7FFFu)));   // exact; NaN stays NaN
}

template <int NT>
__device__ __forceinline__ void count_ge(float ax, const float (&sig)[8], int (&c)[8]) {
#pragma unroll
  for (int i = 0; i < NT; ++i) c[i] += (ax >= sig[i]) ? 1 : 0;
}

template <int NT>
__device__ __forceinline__ void snapshot(const int (&c)[8], int (&cb)[8]) {
#pragma unroll
  for (int i = 0; i < NT; ++i) cb[i] = c[i];
}

// The threshold s as two fp16 copies for comparing |x| two channels at a time:
// |x| is an fp16 value, so |x| >= s exactly when |x| >= ceil_fp16(s) (a NaN s
// stays NaN and is never reached; s above the largest finite half rounds to
// +inf, which only +inf reaches).
__device__ __forceinline__ uint32_t half2_threshold(float s) {
  const uint32_t hb = __half_as_ushort(__float2half_ru(s));
  return hb | (hb << 16);
}

// Two fp16 counters += (|x| >= threshold), one per half (1.0 or 0.0 from an
// ordered compare: NaN counts nowhere). Exact while a counter stays <= 2048.
__device__ __forceinline__ uint32_t count_ge2(uint32_t acc, uint32_t ax2, uint32_t th2) {
  uint32_t ge, out;
  asm("set.ge.f16x2.f16x2 %0, %1, %2;" : "=r"(ge) : "r"(ax2), "r"(th2));
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(out) : "r"(acc), "r"(ge));
  return out;
}

__device__ __forceinline__ int half2_total(uint32_t acc) {
  return (int)(half_bits_to_float(acc) + half_bits_to_float(acc >> 16));
}

// Vector loads of x per thread and batch in the count below: 4 x 8 channels x
// 512 threads covers K <= 16384 in one batch, so the whole count waits for one
// memory round trip (issued right after the kernel's dependency wait).
constexpr int kCountBatch = 4;

// One batch of count_all's loads: thread t's 16-byte groups g0, g0 + 512, ...
// of x (zeros past the end). Only used when x is 16-byte aligned.
__device__ __forceinline__ void count_loads(const uint16_t* __restrict__ x, int K, int g0,
                                            uint4 (&v)[kCountBatch]) {
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  const int g1 = K >> 3;
#pragma unroll
  for (int u = 0; u < kCountBatch; ++u) {
    const int g = g0 + u * kSelThreads;
    v[u] = (g < g1) ? __ldg(xv + g) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// c[i] = #{k : |x_k| >= sig[i]} over this thread's share of [0, K); cb[i] the
// same over k < lo. lo is a multiple of the chunk (so of 8). th2 = the
// thresholds as fp16 pairs; v holds the first batch of loads (count_loads with
// g0 = thread index) when x is aligned. Channels are compared two at a time in
// fp16 and counted in fp16 pairs, flushed to integers after every batch (at
// most 16 per counter).
template <int NT>
__device__ __forceinline__ void count_all(const uint16_t* __restrict__ x, int K, int lo, const float (&sig)[8],
                                          const uint32_t (&th2)[8], uint4 (&v)[kCountBatch], int (&c)[8],
                                          int (&cb)[8]) {
  const int tid = threadIdx.x;
  bool snap = false;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const int g1 = K >> 3, glo = lo >> 3;
#pragma unroll 1
    for (int g0 = tid; g0 < g1; g0 += kCountBatch * kSelThreads) {
      if (g0 != tid) count_loads(x, K, g0, v);
      uint32_t acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0u;
#pragma unroll
      for (int u = 0; u < kCountBatch; ++u) {
        const int g = g0 + u * kSelThreads;
        if (g < g1) {
          if (!snap && g >= glo) {
            snap = true;
#pragma unroll
            for (int i = 0; i < NT; ++i) cb[i] = c[i] + half2_total(acc[i]);
          }
          const uint32_t w[4] = {v[u].x & 0x7FFF7FFFu, v[u].y & 0x7FFF7FFFu, v[u].z & 0x7FFF7FFFu,
                                 v[u].w & 0x7FFF7FFFu};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
#pragma unroll
            for (int i = 0; i < NT; ++i) acc[i] = count_ge2(acc[i], w[q], th2[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < NT; ++i) c[i] += half2_total(acc[i]);
    }
    if (!snap) snapshot<NT>(c, cb);
    const int k = (g1 << 3) + tid;   // at most 7 tail channels, all at or after lo
    if (k < K) count_ge<NT>(abs_half(__ldg(x + k)), sig, c);
  } else {
#pragma unroll 1
    for (int k = tid; k < K; k += kSelThreads) {
      if (!snap && k >= lo) {
        snap = true;
        snapshot<NT>(c, cb);
      }
      count_ge<NT>(abs_half(__ldg(x + k)), sig, c);
    }
    if (!snap) snapshot<NT>(c, cb);
  }
}

template <int NT>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t* __restrict__ x, int K,
                                                             const float* __restrict__ thresholds,
                                                             ClassTable ct, uint8_t* __restrict__ bits,
                                                             int32_t* __restrict__ idx,
                                                             int32_t* __restrict__ offsets) {
  constexpr int NC = NT + 1;
  __shared__ float s_thr[8];
  __shared__ int s_part[2][kSelWarps][8];   // per warp and threshold: channels before the chunk / overall reaching it
  __shared__ int s_cnt[9][32];              // per (round, warp) class counts, then their exclusive prefix
  __shared__ int s_base[9];
  __shared__ uint8_t s_width[9];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lo = blockIdx.x * kSelChunk, hi = min(K, lo + kSelChunk);
  if (tid >= 32 && tid < 32 + NC) s_width[tid - 32] = ct.width[tid - 32];
  pdl_wait();   // x and the thresholds may come from the kernel just before
  if (tid < NT) s_thr[tid] = thresholds[tid];
  uint16_t xo[kSelRounds];
#pragma unroll
  for (int e = 0; e < kSelRounds; ++e) {
    const int k = lo + e * kSelThreads + tid;
    xo[e] = (k < hi) ? __ldg(x + k) : (uint16_t)0;
  }
  // the count's first batch goes out with the chunk's own loads: one round trip
  uint4 xv[kCountBatch];
  if (NT > 0 && (reinterpret_cast<uintptr_t>(x) & 15u) == 0) count_loads(x, K, tid, xv);
  __syncthreads();
  pdl_launch_dependents();
  float sig[8];
  uint32_t th2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sig[i] = (i < NT) ? s_thr[i] : 0.0f;
    th2[i] = (i < NT) ? half2_threshold(sig[i]) : 0u;
  }

  if (NT > 0) {
    int c[8] = {0, 0, 0, 0, 0, 0, 0, 0}, cb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    count_all<NT>(x, K, lo, sig, th2, xv, c, cb);
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const int vb = __reduce_add_sync(0xffffffffu, cb[i]);
      const int vt = __reduce_add_sync(0xffffffffu, c[i]);
      if (lane == 0) {
        s_part[0][warp][i] = vb;
        s_part[1][warp][i] = vt;
      }
    }
  }

  // the class of a channel is the number of thresholds it reaches, whatever
  // their order
  int j[kSelRounds], rank[kSelRounds];
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < kSelRounds; ++e) {
    const int k = lo + e * kSelThreads + tid;
    int jj = 0;
    const float ax = abs_half(xo[e]);
#pragma unroll
    for (int i = 0; i < NT; ++i) jj += (ax >= sig[i]) ? 1 : 0;
    j[e] = (k < hi) ? jj : kNoClass;
    rank[e] = 0;
    if (k < hi) bits[k] = s_width[jj];
#pragma unroll
    for (int cl = 0; cl < NC; ++cl) {
      const uint32_t m = __ballot_sync(0xffffffffu, j[e] == cl);
      if (lane == 0) s_cnt[cl][e * kSelWarps + warp] = __popc(m);
      if (j[e] == cl) rank[e] = __popc(m & lt);
    }
  }
  __syncthreads();
  for (int cl = warp; cl < NC; cl += kSelWarps) {
    const int v = s_cnt[cl][lane];
    int w = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    s_cnt[cl][lane] = w - v;
    // lane i < NT: T = channels reaching threshold i overall, B = before the
    // chunk. Ordered by T descending, the thresholds are in ascending order
    // (equal T means no channel lies between the two thresholds, so B is equal
    // too): position p then holds #{|x| >= sigma_p} for the sorted sigma.
    int T = 0, B = 0;
    if (lane < NT) {
#pragma unroll
      for (int q = 0; q < kSelWarps; ++q) {
        T += s_part[1][q][lane];
        B += s_part[0][q][lane];
      }
    }
    int pos = 0;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const int Ti = __shfl_sync(0xffffffffu, T, i);
      pos += (Ti > T || (Ti == T && i < lane)) ? 1 : 0;
    }
    const bool real = lane < NT;
    // #{class >= c} = #{|x| >= sigma_{c-1}}; channels of class < c precede class c
    int ge_t = K, ge_b = lo, nx_b = 0;
    if (cl > 0) {
      const int src = __ffs(__ballot_sync(0xffffffffu, real && pos == cl - 1)) - 1;
      ge_t = __shfl_sync(0xffffffffu, T, src);
      ge_b = __shfl_sync(0xffffffffu, B, src);
    }
    if (cl < NT) {
      const int src = __ffs(__ballot_sync(0xffffffffu, real && pos == cl)) - 1;
      nx_b = __shfl_sync(0xffffffffu, B, src);
    }
    if (lane == 0) {
      const int first = K - ge_t;
      s_base[cl] = first + ge_b - nx_b;
      if (blockIdx.x == 0) {
        offsets[cl] = first;
        if (cl == NC - 1) offsets[NC] = K;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < kSelRounds; ++e) {
    if (j[e] != kNoClass) {
      const int k = lo + e * kSelThreads + tid;
      idx[s_base[j[e]] + s_cnt[j[e]][e * kSelWarps + warp] + rank[e]] = k;
    }
  }
}

template <int NT>
static cudaError_t launch_select_nt(const cudaLaunchConfig_t& cfg, const uint16_t* x, int K,
                                    const float* thresholds, const ClassTable& ct, uint8_t* bits,
                                    int32_t* idx, int32_t* offsets) {
  return cudaLaunchKernelEx(&cfg, select_kernel<NT>, x, K, thresholds, ct, bits, idx, offsets);
}

cudaError_t launch_select(const uint16_t* x, int K, const float* thresholds, const ClassTable& ct,
                          uint8_t* bits, int32_t* idx, int32_t* offsets, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((K + kSelChunk - 1) / kSelChunk), 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (ct.n - 1) {
    case 0: return launch_select_nt<0>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 1: return launch_select_nt<1>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 2: return launch_select_nt<2>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 3: return launch_select_nt<3>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 4: return launch_select_nt<4>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 5: return launch_select_nt<5>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 6: return launch_select_nt<6>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 7: return launch_select_nt<7>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    case 8: return launch_select_nt<8>(cfg, x, K, thresholds, ct, bits, idx, offsets);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace grinqh
