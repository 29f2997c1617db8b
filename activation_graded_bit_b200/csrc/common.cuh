// Device-side helpers shared by the GRINQH kernels (sm_100a).
//
// Bit-plane word format (see include/grinqh.h): inside plane p (p = 0 is the
// most significant bit of the 8-bit code), 32-bit word w of a tile holds local
// columns 32w..32w+31, and column 32w + 4j + i (j in 0..7, i in 0..3) sits at
// bit (8i + j + 7 - p) mod 32. The placement is chosen so that, for every j,
// the bits a register needs from plane p sit under the mask
// 0x01010101 << ((j + 7 - p) & 7), and one 32-bit rotate by j then moves all
// planes' bits of columns 4j..4j+3 to bit 7-p of byte i. Rebuilding four codes
// therefore costs one LOP3 per plane plus one rotate, instead of one operation
// per bit. This is the "pre-grouping" idea of the paper's Appendix C.1
// (neighbouring weights of the same significance share a 32-bit word, arranged
// offline so that OR/SHIFT rebuilds them), adapted to 1-bit planes.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace grinqh {

constexpr int kPlanes = 8;
constexpr int kGroup = 128;
constexpr int kTileN = 1024;                          // columns per tile
constexpr int kMetaBytes = 4 * (kTileN / kGroup);     // scale/zero words at the head of a record
constexpr int kPlaneBytes = kTileN / 8;               // one plane of one tile row
constexpr int kRecordBytes = kMetaBytes + kPlanes * kPlaneBytes;   // 1056 = 33 sectors of 32 B

// Bit position of local column c (0..31 inside its word) in plane p's word.
__host__ __device__ __forceinline__ int bit_pos(int p, int c) {
  const int j = c >> 2, i = c & 3;
  return (8 * i + j + 7 - p) & 31;
}

// Local column (0..31) stored at bit L of plane p's word (inverse of bit_pos).
__host__ __device__ __forceinline__ int col_at(int p, int L) {
  const int u = (L - 7 + p) & 31;   // = 8i + j
  return 4 * (u & 7) + (u >> 3);
}

// Rebuild the truncated codes of 32 columns from the top B plane words.
// out[j] byte i = top-B bits of column 4j+i, in place (bits 7..8-B), low bits 0.
template <int B>
__device__ __forceinline__ void assemble(const uint32_t (&P)[8], uint32_t (&out)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t t = 0;
#pragma unroll
    for (int p = 0; p < B; ++p) t |= P[p] & (0x01010101u << ((j + 7 - p) & 7));
    out[j] = (j == 0) ? t : __funnelshift_r(t, t, j);
  }
}

// Midpoint term of the nested reconstruction for width b (0 for b = 8):
// 2^(7-b) in every byte (the low 8-b bits of a truncated code are zero, so an
// OR adds it).
__host__ __device__ __forceinline__ uint32_t midpoint_bytes(int b) {
  return b >= 8 ? 0u : 0x01010101u * (1u << (7 - b));
}

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

}  // namespace grinqh
