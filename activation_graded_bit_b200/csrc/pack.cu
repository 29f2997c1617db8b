// Offline packing: b_max-bit RTN per (row, 128-column group) + MSB-first bit
// planes (b_max = 2, 4, 6 or 8), and the test-only decoder of the packed format.
//
// Paper: "GRINQH" Section 3.3 (uniform b_max-bit codes split into significance
// slices, input-major storage), Section 4 (RTN with group size 128) and
// Appendix C.1 (same-significance bits of neighbouring weights in one 32-bit
// word, grouped offline so the kernel rebuilds codes with OR/SHIFT).
#include <cstdint>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace grinqh {

// fp64 -> binary16, round to nearest even, in one conversion (no fp32 detour).
__device__ __forceinline__ uint16_t f64_to_f16_rn(double v) {
  unsigned short h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return h;
}

__device__ __forceinline__ double f16_to_f64(uint16_t h) {
  return (double)__half2float(__ushort_as_half(h));
}

// One CTA per (row k, tile t): 8 warps, warp g handles the tile's group g
// (128 columns), then 64 threads per plane pair build the b_max/2 pairs of
// plane words of the record.
__global__ void __launch_bounds__(256) pack_kernel(const float* __restrict__ W, int K, int N, int n_tiles,
                                                   int n_groups, int b_max, uint8_t* __restrict__ packed) {
  __shared__ uint8_t codes[kTileN];
  const int k = blockIdx.x, t = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gl = t * (kTileN / kGroup) + warp;     // global group index
  const int c0 = gl * kGroup;                      // first column of the group
  const float* row = W + (size_t)k * N;
  const int rbytes = record_bytes_for(b_max);
  const double levels = (double)((1 << b_max) - 1);
  const size_t ri = (size_t)k * n_tiles + t;
  uint8_t* rec = packed + ri * rbytes;                                                    // its planes
  uint32_t* meta = reinterpret_cast<uint32_t*>(packed + meta_offset_for(K, n_tiles, b_max) + ri * kMetaBytes);

  float v[4];
  float mn = INFINITY, mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int n = c0 + lane + 32 * e;
    v[e] = (n < N) ? row[n] : 0.0f;
    if (n < N) { mn = fminf(mn, v[e]); mx = fmaxf(mx, v[e]); }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const bool live = gl < n_groups;
  double s = 1.0, z = 0.0;
  uint16_t sb = 0, zb = 0;
  if (live) {
    const double range = __dsub_rn((double)mx, (double)mn);
    sb = f64_to_f16_rn(__ddiv_rn(range, levels));
    s = f16_to_f64(sb);
    if (s == 0.0) { sb = 0x3C00; s = 1.0; }
    if (isinf(s)) { sb = 0x7BFF; s = 65504.0; }
    z = rint(__ddiv_rn(-(double)mn, s));
    z = __dadd_rn(fmin(fmax(z, 0.0), levels), 0.0);   // -0 -> +0
    zb = f64_to_f16_rn(z);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int n = c0 + lane + 32 * e;
    uint8_t q = 0;
    if (live && n < N) {
      double qv = __dadd_rn(rint(__ddiv_rn((double)v[e], s)), z);
      qv = fmin(fmax(qv, 0.0), levels);
      q = (uint8_t)qv;
    }
    codes[warp * kGroup + lane + 32 * e] = q;
  }
  if (lane == 0) meta[warp] = live ? ((uint32_t)sb | ((uint32_t)zb << 16)) : 0u;
  __syncthreads();

  // thread -> (pair s, word wi): b_max/2 plane pairs x 64 words for a
  // 1024-column tile; word wi is half wi & 1 of lane wi >> 1's 32 columns;
  // plane p holds bit b_max-1-p of the code
  const int sp = threadIdx.x >> 6, wi = threadIdx.x & 63;
  if (2 * sp >= b_max) return;
  const int cbase = 32 * (wi >> 1) + 16 * (wi & 1);
  uint32_t word = 0;
#pragma unroll 8
  for (int L = 0; L < 32; ++L) {
    int c16, l;
    pair_col_at(sp, L, c16, l);
    const int p = 2 * sp + l;
    word |= (uint32_t)((codes[cbase + c16] >> (b_max - 1 - p)) & 1u) << L;
  }
  reinterpret_cast<uint32_t*>(rec + sp * kPairBytes)[wi] = word;
}

// Decoder: one warp per (row, tile) record, 8 records per CTA. The planes are
// rebuilt in the 8-bit frame (plane p at bit 7-p), then shifted down to the
// b_max-bit code with the midpoint 2^(b_max-B-1) of a width B < b_max.
template <int B>
__device__ __forceinline__ void decode_word(const uint8_t* rec, int w, int b_max, uint32_t (&R)[8]) {
  uint32_t P[8];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const bool used = 2 * s < B;   // pair s holds planes 2s, 2s+1
    const uint32_t* pw = reinterpret_cast<const uint32_t*>(rec + s * kPairBytes);
    P[2 * s] = used ? pw[2 * w] : 0u;
    P[2 * s + 1] = used ? pw[2 * w + 1] : 0u;
  }
  assemble<B>(P, R);
  const int sh = 8 - b_max;
  const uint32_t keep = 0x01010101u * ((1u << b_max) - 1u);
  const uint32_t mid = (B < b_max) ? 0x01010101u * (1u << (b_max - B - 1)) : 0u;
#pragma unroll
  for (int j = 0; j < 8; ++j) R[j] = ((R[j] >> sh) & keep) | mid;
}

__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t* __restrict__ packed,
                                                     const uint8_t* __restrict__ bits, int K, int N,
                                                     int n_tiles, int b_max, uint8_t* __restrict__ codes) {
  const int t = blockIdx.y;
  const int k = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int w = threadIdx.x & 31;
  if (k >= K) return;
  const int b = min(bits ? (int)bits[k] : b_max, b_max);   // a width above b_max decodes as b_max
  const uint8_t* rec = packed + ((size_t)k * n_tiles + t) * record_bytes_for(b_max);
  uint32_t R[8];
  switch (b) {
    case 1: decode_word<1>(rec, w, b_max, R); break;
    case 2: decode_word<2>(rec, w, b_max, R); break;
    case 3: decode_word<3>(rec, w, b_max, R); break;
    case 4: decode_word<4>(rec, w, b_max, R); break;
    case 5: decode_word<5>(rec, w, b_max, R); break;
    case 6: decode_word<6>(rec, w, b_max, R); break;
    case 7: decode_word<7>(rec, w, b_max, R); break;
    case 8: decode_word<8>(rec, w, b_max, R); break;
    default:
#pragma unroll
      for (int j = 0; j < 8; ++j) R[j] = 0u;
  }
  const int n0 = t * kTileN + 32 * w;
  uint8_t* out = codes + (size_t)k * N;
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = n0 + 4 * j + i;
      if (n < N) out[n] = (uint8_t)(R[j] >> (8 * i));
    }
}

// Full-width dequantisation for the prefill product: one warp per (row, tile)
// record, 8 records per CTA; lane w rebuilds its 32 columns at b_max and writes
// w_hat = s (q - z) rounded once to binary16 (the fp32 product of an 11-bit
// scale and a 9-bit code difference is exact). A lane's 32 columns are 64
// contiguous bytes, written as four 16-byte stores when the row allows it.
template <int B>
__device__ __forceinline__ void dequant_record(const uint8_t* rec, const uint8_t* meta, int w, int k, int N, int n0,
                                               __half* __restrict__ out) {
  uint32_t R[8];
  decode_word<B>(rec, w, B, R);
  const uint32_t m = reinterpret_cast<const uint32_t*>(meta)[w >> 2];   // this lane's group's scale | zero
  const float s = __half2float(__ushort_as_half((unsigned short)(m & 0xFFFFu)));
  const float z = __half2float(__ushort_as_half((unsigned short)(m >> 16)));
  __half2 h[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float c0 = (float)(R[j] & 0xFFu), c1 = (float)((R[j] >> 8) & 0xFFu);
    const float c2 = (float)((R[j] >> 16) & 0xFFu), c3 = (float)(R[j] >> 24);
    h[2 * j] = __floats2half2_rn(s * (c0 - z), s * (c1 - z));
    h[2 * j + 1] = __floats2half2_rn(s * (c2 - z), s * (c3 - z));
  }
  __half* row = out + (size_t)k * N;
  if (n0 + 32 <= N && (N & 7) == 0) {
    uint4* dst = reinterpret_cast<uint4*>(row + n0);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      dst[q] = make_uint4(*reinterpret_cast<const uint32_t*>(&h[4 * q]), *reinterpret_cast<const uint32_t*>(&h[4 * q + 1]),
                          *reinterpret_cast<const uint32_t*>(&h[4 * q + 2]), *reinterpret_cast<const uint32_t*>(&h[4 * q + 3]));
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (n0 + c < N) row[n0 + c] = (c & 1) ? __high2half(h[c >> 1]) : __low2half(h[c >> 1]);
  }
}

__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ packed, int K, int N, int n_tiles,
                                                      int b_max, __half* __restrict__ out) {
  const int t = blockIdx.y;
  const int k = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int w = threadIdx.x & 31;
  if (k >= K) return;
  const size_t ri = (size_t)k * n_tiles + t;
  const uint8_t* rec = packed + ri * record_bytes_for(b_max);
  const uint8_t* meta = packed + meta_offset_for(K, n_tiles, b_max) + ri * kMetaBytes;
  const int n0 = t * kTileN + 32 * w;
  if (n0 >= N) return;
  switch (b_max) {
    case 2: dequant_record<2>(rec, meta, w, k, N, n0, out); break;
    case 4: dequant_record<4>(rec, meta, w, k, N, n0, out); break;
    case 6: dequant_record<6>(rec, meta, w, k, N, n0, out); break;
    default: dequant_record<8>(rec, meta, w, k, N, n0, out); break;
  }
}

cudaError_t launch_dequant(const void* packed, int K, int N, int n_tiles, int b_max, uint16_t* out,
                           cudaStream_t st) {
  dim3 grid((K + 7) / 8, n_tiles);
  dequant_kernel<<<grid, 256, 0, st>>>((const uint8_t*)packed, K, N, n_tiles, b_max, reinterpret_cast<__half*>(out));
  return cudaGetLastError();
}

cudaError_t launch_pack(const float* W, int K, int N, int n_tiles, int n_groups, int b_max, void* packed,
                        cudaStream_t st) {
  dim3 grid(K, n_tiles);
  pack_kernel<<<grid, 256, 0, st>>>(W, K, N, n_tiles, n_groups, b_max, (uint8_t*)packed);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const void* packed, const uint8_t* bits, int K, int N, int n_tiles, int b_max,
                          uint8_t* codes, cudaStream_t st) {
  dim3 grid((K + 7) / 8, n_tiles);
  unpack_kernel<<<grid, 256, 0, st>>>((const uint8_t*)packed, bits, K, N, n_tiles, b_max, codes);
  return cudaGetLastError();
}

// Planes of codes given by the caller (nested table codes, or any b_max-bit
// codes quantised elsewhere): one CTA per (row k, tile t), the tile's codes
// staged in shared memory (bits above b_max dropped, columns past N zero), the
// record's scale/zero words written as zero, then the plane-pair words as in
// pack_kernel.
__global__ void __launch_bounds__(256) pack_codes_kernel(const uint8_t* __restrict__ codes, int K, int N,
                                                         int n_tiles, int b_max, uint8_t* __restrict__ packed) {
  __shared__ uint8_t tile[kTileN];
  const int k = blockIdx.x, t = blockIdx.y;
  const size_t ri = (size_t)k * n_tiles + t;
  uint8_t* rec = packed + ri * record_bytes_for(b_max);
  uint32_t* meta = reinterpret_cast<uint32_t*>(packed + meta_offset_for(K, n_tiles, b_max) + ri * kMetaBytes);
  const uint32_t keep = (1u << b_max) - 1u;
  for (int e = threadIdx.x; e < kTileN; e += 256) {
    const int n = t * kTileN + e;
    tile[e] = (n < N) ? (uint8_t)(codes[(size_t)k * N + n] & keep) : (uint8_t)0;
  }
  if (threadIdx.x < kMetaBytes / 4) meta[threadIdx.x] = 0u;
  __syncthreads();
  const int sp = threadIdx.x >> 6, wi = threadIdx.x & 63;
  if (2 * sp >= b_max) return;
  const int cbase = 32 * (wi >> 1) + 16 * (wi & 1);
  uint32_t word = 0;
#pragma unroll 8
  for (int L = 0; L < 32; ++L) {
    int c16, l;
    pair_col_at(sp, L, c16, l);
    word |= (uint32_t)((tile[cbase + c16] >> (b_max - 1 - (2 * sp + l))) & 1u) << L;
  }
  reinterpret_cast<uint32_t*>(rec + sp * kPairBytes)[wi] = word;
}

cudaError_t launch_pack_codes(const uint8_t* codes, int K, int N, int n_tiles, int b_max, void* packed,
                              cudaStream_t st) {
  dim3 grid(K, n_tiles);
  pack_codes_kernel<<<grid, 256, 0, st>>>(codes, K, N, n_tiles, b_max, (uint8_t*)packed);
  return cudaGetLastError();
}

}  // namespace grinqh
