// Device-side helpers shared by the GRINQH kernels (sm_100a).
//
// Packed layout (see include/grinqh.h): the planes of every (row k, column
// tile t) record come first, record k * n_tiles + t at byte
// (k * n_tiles + t) * 128 * b_max (a multiple of 256), and the 32 bytes of
// scale/zero words of every record follow in a separate array. Inside a
// record, planes 2s and 2s+1 (plane 0 is the most significant bit of the code)
// share 256 bytes, "pair s". Lane w of a warp owns words 2w (local columns
// 32w..32w+15) and 2w+1 (columns 32w+16..32w+31) of every pair. In either word, local column
// 4j' + i of the half (j' in 0..3, i in 0..3) of plane 2s + l sits at bit
// (8i + 2j' + 7 - 2s - l) mod 32. The placement is chosen so that the bits a
// register of four codes needs from a pair sit under one rotated mask
// (0x03030303 rotated left by 2j' + 6 - 2s), and one 32-bit rotate right by
// 2j' then moves every plane's bit of columns 4j'..4j'+3 to bit 7-p of byte i.
// Rebuilding four codes therefore costs one LOP3 per two planes plus one
// rotate, and a lane reads two planes with one 8-byte load. This is the
// "pre-grouping" idea of the paper's Appendix C.1 (neighbouring weights of the
// same significance share a 32-bit word, arranged offline so that OR/SHIFT
// rebuilds them), with its 2-bit segments; odd widths take the top plane of
// their last pair under a one-plane mask.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>

namespace grinqh {

constexpr int kPlanes = 8;
constexpr int kGroup = 128;
constexpr int kTileN = 1024;                          // columns per tile
constexpr int kMetaBytes = 4 * (kTileN / kGroup);     // scale/zero words of one (row, tile) record
constexpr int kPlaneBytes = kTileN / 8;               // one plane of one tile row
constexpr int kPairBytes = 2 * kPlaneBytes;           // two planes of one tile row

// Plane bytes of a (row, tile) record that stores b_max planes: b_max / 2 plane
// pairs of 256 bytes.
__host__ __device__ constexpr int record_bytes_for(int b_max) { return b_max * kPlaneBytes; }

// Byte offset of the scale/zero words in a packed layer: after every record's planes.
__host__ __device__ constexpr size_t meta_offset_for(int K, int n_tiles, int b_max) {
  return (size_t)K * (size_t)n_tiles * (size_t)record_bytes_for(b_max);
}

// The column (0..15 inside the half) and plane offset l stored at bit L of a
// pair-s word (the inverse of the placement above: column 4j'+i of plane 2s+l
// at bit (8i + 2j' + 7 - 2s - l) mod 32).
__host__ __device__ __forceinline__ void pair_col_at(int s, int L, int& c16, int& l) {
  const int u = (L - 7 + 2 * s) & 31;   // 8i + 2j' - l (mod 32)
  l = u & 1;
  const int v = (u + l) & 31;           // 8i + 2j'
  c16 = 4 * ((v & 7) >> 1) + (v >> 3);
}

__host__ __device__ constexpr uint32_t rotl32(uint32_t x, int k) {
  return (k & 31) ? ((x << (k & 31)) | (x >> (32 - (k & 31)))) : x;
}

// OR both planes of pair S into the eight code registers (A: this lane's low
// half word, B: its high half word), or only the top plane of the pair.
template <int S>
__device__ __forceinline__ void merge_pair(uint32_t A, uint32_t B, uint32_t (&T)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) T[j] |= ((j < 4) ? A : B) & rotl32(0x03030303u, 2 * (j & 3) + 6 - 2 * S);
}
template <int S>
__device__ __forceinline__ void merge_pair_top(uint32_t A, uint32_t B, uint32_t (&T)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) T[j] |= ((j < 4) ? A : B) & rotl32(0x01010101u, 2 * (j & 3) + 7 - 2 * S);
}

// After the merges: byte i of out[j] = top bits of column 4j+i, in place.
__device__ __forceinline__ void finish_codes(const uint32_t (&T)[8], uint32_t (&out)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) out[j] = (j & 3) ? __funnelshift_r(T[j], T[j], 2 * (j & 3)) : T[j];
}

// Rebuild the truncated codes of a lane's 32 columns for a width B known at
// compile time. P[2s], P[2s+1] = the lane's two words of pair s.
template <int B>
__device__ __forceinline__ void assemble(const uint32_t (&P)[8], uint32_t (&out)[8]) {
  uint32_t T[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) T[j] = 0u;
  if (B >= 2) merge_pair<0>(P[0], P[1], T);
  if (B >= 4) merge_pair<1>(P[2], P[3], T);
  if (B >= 6) merge_pair<2>(P[4], P[5], T);
  if (B >= 8) merge_pair<3>(P[6], P[7], T);
  if (B == 1) merge_pair_top<0>(P[0], P[1], T);
  if (B == 3) merge_pair_top<1>(P[2], P[3], T);
  if (B == 5) merge_pair_top<2>(P[4], P[5], T);
  if (B == 7) merge_pair_top<3>(P[6], P[7], T);
  finish_codes(T, out);
}

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

}  // namespace grinqh
