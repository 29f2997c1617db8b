// The graded bit-plane VMM: y = x . W_hat over the top-b_k planes of each row.
//
// Paper: "GRINQH" Fig. 2 and Section 3.3: for every input channel k with
// b_k > 0 only the b_k most significant slices of row k move from DRAM to the
// SM; the row is rebuilt on chip and channels with b_k = 0 are bypassed. The
// rebuilt weight is w_hat = s * (code - z), code = c_b * 2^(8-b) + 2^(7-b) for
// b < 8 (Section 3.3, bias correction) and q for b = 8.
//
// Work split. The grid is (column tile t, row split r). Every CTA walks the same
// class-ordered channel list from grinqh_select; the list is cut into
// gridDim.y pieces of equal DRAM cost (16 B of scale/zero + 64 B per plane for a
// 512-column tile), computed in each CTA from the class offsets alone. Because
// classes are stored in ascending width and only the first can be 0, the rows
// to read form one contiguous stretch of the list.
//
// Arithmetic. Per row, per 128-column group: a = x_k * s_kg is exact in fp32
// (two 11-bit significands). The truncated code c (low bits zero) is turned
// into a float exactly, and the row adds a * c to the column accumulators and
// a * (mid_b - z) once to a per-thread constant, since every column of a thread
// shares one group.
//
// Reduction. 16 row lanes of a CTA are summed in shared memory; CTAs of one
// column tile add into an fp32 accumulator in the workspace with L2 atomics.
// The last CTA of a tile to finish (a ticket counter, no waiting) copies the
// tile to y and clears the accumulator and the ticket, so the workspace is
// zero again for the next call.
#include <cstdint>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace grinqh {

constexpr int kTile = 512;                 // columns per tile
constexpr int kWords = kTile / 32;         // plane words per tile row
constexpr int kThreads = 256;
constexpr int kLanes = kThreads / kWords;  // rows processed side by side

__device__ __forceinline__ float byte_as_float(uint32_t r, int i) {
  // 0x4B000000 | byte is the float 2^23 + byte; subtracting 2^23 is exact
  const uint32_t f = __byte_perm(r, 0x4B000000u, 0x7650u | (uint32_t)i);
  return __uint_as_float(f) - 8388608.0f;
}

// cost of one row of class width b, in 16-byte units of a 512-column tile
__device__ __forceinline__ long long row_cost(int b) { return b > 0 ? 1 + 4 * b : 0; }

// First list position whose cumulative cost, scaled by R, reaches X.
__device__ long long split_point(const int* off, const ClassTable& ct, int first_active, int K,
                                 long long X, int R) {
  long long C = 0;   // cost before the current class
  for (int j = first_active; j < ct.n; ++j) {
    const long long c = row_cost(ct.width[j]);
    const long long cnt = off[j + 1] - off[j];
    if ((C + cnt * c) * R >= X) {
      const long long need = X - C * R;            // > 0 unless X <= C*R
      long long m = need <= 0 ? 0 : (need + c * R - 1) / (c * R);
      if (m > cnt) m = cnt;
      return off[j] + m;
    }
    C += cnt * c;
  }
  return K;
}

template <int B>
__device__ __forceinline__ void process_rows(const VmmArgs& a, int t, int lo, int hi, int lane_row,
                                             int w, float (&acc)[32], float& cacc) {
  const int K = a.K;
  const uint32_t* plane_base = a.planes + (size_t)t * K * (kTile / 4) + w;
  const uint32_t* meta_base = a.meta + t * (kTile / kGroup) + (w >> 2);
  const float mid = (B >= 8) ? 0.0f : (float)(1 << (7 - B));
  for (int i = lo + lane_row; i < hi; i += kLanes) {
    const int k = a.idx[i];
    const uint32_t m = __ldg(meta_base + (size_t)k * a.meta_stride);
    const float xk = __half2float(__ushort_as_half(__ldg(a.x + k)));
    const float s = half_bits_to_float(m);
    const float z = half_bits_to_float(m >> 16);
    const float av = xk * s;   // exact: 11-bit x 11-bit significands
    uint32_t P[8];
    const uint32_t* rec = plane_base + (size_t)k * (kTile / 4);
#pragma unroll
    for (int p = 0; p < 8; ++p) P[p] = (p < B) ? __ldg(rec + p * kWords) : 0u;
    uint32_t R[8];
    assemble<B>(P, R);
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) acc[4 * j + i4] = fmaf(av, byte_as_float(R[j], i4), acc[4 * j + i4]);
    cacc = fmaf(av, mid - z, cacc);
  }
}

__global__ void __launch_bounds__(kThreads) vmm_kernel(const VmmArgs a) {
  __shared__ int s_off[10];
  __shared__ float s_red[kLanes][kTile + 16];
  __shared__ int s_last;
  const int t = blockIdx.x, r = blockIdx.y, R = gridDim.y;
  const int tid = threadIdx.x;
  const int lane_row = tid / kWords, w = tid % kWords;
  const ClassTable& ct = a.ct;
  if (tid <= ct.n) s_off[tid] = a.offsets[tid];
  __syncthreads();

  const int first_active = (ct.width[0] == 0) ? 1 : 0;
  long long W = 0;
  for (int j = first_active; j < ct.n; ++j) W += (long long)(s_off[j + 1] - s_off[j]) * row_cost(ct.width[j]);
  const int lo = (int)split_point(s_off, ct, first_active, a.K, W * r, R);
  const int hi = (int)split_point(s_off, ct, first_active, a.K, W * (r + 1), R);

  float acc[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) acc[c] = 0.0f;
  float cacc = 0.0f;
  for (int j = first_active; j < ct.n; ++j) {
    const int s0 = max(lo, s_off[j]), s1 = min(hi, s_off[j + 1]);
    if (s0 >= s1) continue;
    switch (ct.width[j]) {
      case 1: process_rows<1>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 2: process_rows<2>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 3: process_rows<3>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 4: process_rows<4>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 5: process_rows<5>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 6: process_rows<6>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 7: process_rows<7>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      case 8: process_rows<8>(a, t, s0, s1, lane_row, w, acc, cacc); break;
      default: break;
    }
  }

  // column (32w + c) of the tile -> shared slot [lane_row][c*16 + w]
#pragma unroll
  for (int c = 0; c < 32; ++c) s_red[lane_row][c * kWords + w] = acc[c] + cacc;
  __syncthreads();
  float* accum = a.accum + (size_t)t * kTile;
  if (hi > lo) {
    for (int e = tid; e < kTile; e += kThreads) {
      float v = 0.0f;
#pragma unroll
      for (int l = 0; l < kLanes; ++l) v += s_red[l][e];
      const int c = e / kWords, ww = e % kWords;
      atomicAdd(accum + 32 * ww + c, v);
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(a.counters + t, 1u);
    s_last = (prev == (unsigned)(R - 1));
    __threadfence();
  }
  __syncthreads();
  if (s_last) {
    for (int e = tid; e < kTile; e += kThreads) {
      const int n = t * kTile + e;
      const float v = __ldcg(accum + e);
      if (n < a.N) a.y[n] = v;
      __stcg(accum + e, 0.0f);
    }
    if (tid == 0) a.counters[t] = 0u;
  }
}

size_t vmm_workspace_bytes(int n_tiles, int tile_n) {
  const size_t acc = (size_t)n_tiles * tile_n * sizeof(float);
  const size_t cnt = (size_t)n_tiles * sizeof(uint32_t);
  return (acc + cnt + 15) & ~(size_t)15;
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

cudaError_t launch_vmm(const VmmArgs& a, cudaStream_t st) {
  const int nsm = sm_count();
  int R = (2 * nsm + a.n_tiles - 1) / a.n_tiles;
  if (R < 1) R = 1;
  if (R > 1024) R = 1024;
  dim3 grid(a.n_tiles, R);
  vmm_kernel<<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace grinqh
