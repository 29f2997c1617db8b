// The graded bit-plane VMM: y = x . W_hat over the top-b_k planes of each row.
//
// Paper: "GRINQH" Fig. 2 and Section 3.3: for every input channel k with
// b_k > 0 only the b_k most significant slices of row k move from DRAM to the
// SM; the row is rebuilt on chip; channels with b_k = 0 are bypassed. The
// rebuilt weight is w_hat = s * (code - z), code = c_b * 2^(8-b) + 2^(7-b) for
// b < 8 (the bias correction of Section 3.3) and q for b = 8.
//
// Work split. The grid is (column tile t of 1024 columns, row split r), one CTA
// per SM. Every CTA walks the class-ordered channel list written by
// grinqh_select: CTA r of R takes list positions r, r + R, r + 2R, ..., so
// every CTA gets the same mix of widths (equal DRAM bytes and equal arithmetic
// per CTA), and skips the width-0 class (classes are stored by ascending width
// and only the first can be 0, so its positions are a prefix of every CTA's
// sequence). The CTA loads its first channel indices together with the class
// offsets, in one memory round trip.
//
// Data movement. Each of the 16 warps takes rows h, h+16, ... of its CTA. Lane
// w of a warp owns columns 32w..32w+31 of the tile, so for a row of width b it
// needs its two words of each of plane pairs 0..ceil(b/2)-1 (one 8-byte load
// per pair: 256 contiguous, 256-byte-aligned bytes per pair across the warp,
// one coalesced request) and the scale/zero word of its 128-column group (the
// scale/zero words of all records sit in their own array, so the plane records
// are whole 256-byte units and no DRAM sector is shared between records). The lanes load
// those words straight into registers with plain read-only loads, kDepth rows
// ahead of the one they are rebuilding: a software pipeline in registers, with
// no shared-memory staging and no barriers. On this part that reads scattered
// 300..1100-byte rows faster than bulk (TMA) copies, whose completion rate per
// issuing warp, not their size, limits the bandwidth for rows this short. The
// planes and scale/zero words of the kL2Ahead rows beyond the pipeline are
// requested into L2 (one 128-byte line per lane, no register), so the register
// loads hit L2
// instead of DRAM. With those requests a pipeline of three rows is enough, and
// the registers it frees go to the compiler's scheduling (measured: 3 rows in
// flight 13% faster than 6 on the 14336 x 4096 layer). Blocks of kDepth rows
// whose loads and requests all exist run without per-row tests; the loads of
// narrower rows are switched off by predicates, not branches.
//
// Arithmetic per row and thread. The row's coefficient a = x_k * s is one
// mixed-precision FMA of the two binary16 values (exact in fp32), and
// z - mid one mixed-precision add. The plane pairs are merged into 8 registers
// of 4 truncated codes each (one LOP3 per pair plus one rotate, thanks to the
// bit order chosen at pack time); the merge enters one fall-through sequence at
// the last pair, so all widths share one copy of the code. Codes become floats
// without a per-code integer extraction: a byte-permute puts two codes c1:c0 in
// the low 16 bits of an otherwise zero word, i.e. the subnormal float
// (256 c1 + c0) 2^-149; a multiply by 2^-8 rounded toward zero leaves exactly
// hi = c1 2^-149 (the subnormal grid is 2^-149) and one FMA gives
// lo = c0 2^-149 = X - 256 hi, both exact and on the FP32 pipe (B200 runs
// FFMA with subnormal operands at full rate, while byte extraction would run on
// the half-rate integer pipe). Both halves take the same coefficient a 2^95,
// so the accumulators hold a * code * 2^-54 (no overflow for |a| <= 2^32, no
// precision loss for the sizes that matter). The per-row constant
// a * (mid_b - z) goes to one scalar per thread, since all 32 columns of a
// thread share one 128-column group.
//
// Reduction. Each warp stores its 1024 column sums into shared memory as soon
// as its own rows are done (the buffer is not shared with the row list); after
// one barrier the CTA sums the 16 warps into one 1024-column partial, stored
// with plain coalesced stores into the workspace as partial[r][column]. A
// second kernel, chained with programmatic dependent launch, sums the R
// partials of every column in a fixed order (every load of a column in flight
// at once) and overwrites y, so repeated calls give the same bits. (Finishing
// the sum inside this kernel, with vector L2 reductions into a per-tile
// accumulator and the last CTA to arrive writing y, measured no faster, and
// its order of additions varies from call to call.) With a single row split
// (R = 1) the CTA writes y directly and no second kernel runs. A batch of
// tokens (grinqh_select_vmm_batch) adds a grid dimension: token z reads
// x + z K and has its own set of partials and its own y row.
#include <cstdint>
#include <cuda_fp16.h>
#include <atomic>
#include <mutex>

#include "async.cuh"
#include "common.cuh"
#include "kernels.h"

namespace grinqh {

constexpr int kWords = kTileN / 32;              // plane words per tile row (32)
constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kDepth = 3;                        // rows in flight per warp (register slots)
constexpr int kL2Ahead = 3;                      // rows beyond those whose records are prefetched to L2
constexpr int kIdxCap = 16384;                   // rows of a CTA staged per pass (64 KB)
constexpr int kFusedMaxK = kIdxCap;              // fused grading: every CTA's rows fit one pass
constexpr int kRedPitch = 33;                    // column c of word w at c*33 + w: conflict-free both ways
constexpr int kRedStride = 32 * kRedPitch + 16;  // floats per warp in the reduction buffer

struct __align__(16) VmmSmem {
  struct {
    uint32_t rows[kIdxCap];                      // k | b << 24 of this CTA's rows, one pass
    float red[kWarps * kRedStride];              // per-warp column sums, written as each warp finishes
  } u;
  int off[10];
  int width[9];
  int wcnt[2][kWarps];                           // fused grading: rows kept per warp, two rounds
};

// One row in flight: this lane's scale/zero word, its two words of each plane
// pair (p[2s], p[2s+1]) and x_k.
struct RowRegs {
  uint32_t m;
  uint32_t p[8];
  uint32_t xh;
  uint32_t b;
};

// Per-thread constants of the row addressing. A row's record index
// rec = k * n_tiles + t is below 2^26 (a valid layout has K * N <= 2^34), so one
// wide multiply-add gives each address: the planes of record rec start at
// packed + rec * 128 b_max, its scale/zero words at packed + meta_offset + 32 rec.
struct RowAddr {
  const uint8_t* meta;    // this lane's scale/zero word within record 0's
  const uint8_t* pairs;   // this lane's two words of pair 0 within record 0
  const uint8_t* line;    // the L2 line this lane requests for record 0: plane line `lane` (lanes < b_max)
                          // or the scale/zero words (lane b_max)
  uint32_t line_mul;      // bytes per record in the array `line` points into
  uint32_t lane;
  uint32_t nt, t;         // column tiles, this CTA's tile
};

__device__ __forceinline__ RowAddr row_addr(const VmmArgs& a, int t, int w) {
  const uint8_t* meta0 = a.packed + a.meta_offset;
  RowAddr ra;
  ra.meta = meta0 + 4 * (w >> 2);
  ra.pairs = a.packed + 8 * w;
  ra.lane = (uint32_t)w;
  if (w < a.b_max) {
    ra.line = a.packed + 128 * w;
    ra.line_mul = (uint32_t)record_bytes_for(a.b_max);
  } else {
    ra.line = meta0;
    ra.line_mul = (uint32_t)kMetaBytes;
  }
  ra.nt = (uint32_t)a.n_tiles;
  ra.t = (uint32_t)t;
  return ra;
}

// Read-only load that skips L1 allocation (every weight word is read once).
__device__ __forceinline__ uint32_t ld_stream(const void* ptr) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}
// Two words at a constant byte offset (folded into the instruction, so a row's
// plane-pair loads share one address register).
template <int kOff>
__device__ __forceinline__ void ld_stream2_at(const void* ptr, uint32_t& lo, uint32_t& hi) {
  asm volatile("ld.global.nc.L1::no_allocate.v2.b32 {%0, %1}, [%2+%3];" : "=r"(lo), "=r"(hi) : "l"(ptr), "n"(kOff));
}
// The same load under a predicate instead of a branch; when it is off the
// registers keep what they held.
template <int kOff>
__device__ __forceinline__ void ld_stream2_at_if(bool on, const void* ptr, uint32_t& lo, uint32_t& hi) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %3, 0;\n\t"
      "@p ld.global.nc.L1::no_allocate.v2.b32 {%0, %1}, [%2+%4];\n\t}"
      : "+r"(lo), "+r"(hi)
      : "l"(ptr), "r"((uint32_t)on), "n"(kOff));
}

// Per-row coefficient for codes of kBmax bits, rebuilt in the 8-bit frame
// (plane p at bit 7-p, so a code c of kBmax bits reads as c 2^(8-kBmax)):
// A = a 2^(87+kBmax) for codes held as c 2^-149, so the products carry
// a * c 2^-54 in kBmax-bit units; the row's constant a * (mid - z) is added to
// cacc (mid = 2^(kBmax-b-1) for b < kBmax, 0 at b = kBmax, in the units of z).
// a = x * s is one mixed-precision FMA of the binary16 values (exact in fp32)
// and z - mid one mixed-precision add (exact).
template <int kBmax>
__device__ __forceinline__ void row_coef(uint32_t m, uint32_t xh, float mid, float& A, float& cacc) {
  float a, zt;
  asm("{\n\t.reg .b16 s, z;\n\tmov.b32 {s, z}, %2;\n\t"
      "fma.rn.f32.f16 %0, %3, s, 0f00000000;\n\t"
      "add.rn.f32.f16 %1, z, %4;\n\t}"
      : "=f"(a), "=f"(zt)
      : "r"(m), "h"((unsigned short)xh), "f"(-mid));
  cacc = fmaf(-a, zt, cacc);
  A = a * ((float)(1ull << (23 + kBmax)) * 0x1p64f);
}

// The bin midpoint of width b for codes of kBmax bits, 0 at full width.
template <int kBmax>
__device__ __forceinline__ constexpr float midpoint(int b) {
  return b >= kBmax ? 0.0f : (float)(1u << (kBmax - b - 1));
}

// acc += codes * A for the 32 columns held in R (one row): acc[2j] holds
// columns 4j, 4j+2 and acc[2j+1] columns 4j+1, 4j+3.
__device__ __forceinline__ void fma_codes(const uint32_t (&R)[8], float As, float2 (&acc)[16]) {
  const float2 A = make_float2(As, As);
  const float2 S8 = make_float2(0x1p-8f, 0x1p-8f);
  const float2 M256 = make_float2(-256.0f, -256.0f);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // X.x = codes of columns 4j+1 : 4j, X.y = columns 4j+3 : 4j+2, as subnormals
    const float2 X = make_float2(__uint_as_float(__byte_perm(R[j], 0u, 0x4410u)),
                                 __uint_as_float(__byte_perm(R[j], 0u, 0x4432u)));
    const float2 hi = __fmul2_rz(X, S8);         // c_hi 2^-149 (the c_lo part is cut off)
    const float2 lo = __ffma2_rn(hi, M256, X);   // c_lo 2^-149
    acc[2 * j] = __ffma2_rn(A, lo, acc[2 * j]);
    acc[2 * j + 1] = __ffma2_rn(A, hi, acc[2 * j + 1]);
  }
}

// Issue the loads of one row (k | b << 24, b >= 1) into r: the scale/zero word
// of this lane's group, x_k (a broadcast 2-byte load) and this lane's two words
// of plane pairs 0..ceil(b/2)-1 of the row's record (each an 8-byte load, a
// coalesced 256-byte request across the warp). Pairs 1..3 are loaded under a
// predicate: a narrow row reads no pair it does not use, and no branch is taken.
// Every row that reaches the loop has b >= 1 (the width-0 class is never staged).
template <int kBmax>
__device__ __forceinline__ void load_row(const uint16_t* __restrict__ x, const RowAddr& ra, uint32_t info,
                                         RowRegs& r) {
  const uint32_t k = info & 0xFFFFFFu, b = info >> 24;
  const uint32_t rec = k * ra.nt + ra.t;
  r.b = b;
  r.m = ld_stream(ra.meta + (size_t)rec * kMetaBytes);
  r.xh = __ldg(x + k);
  const uint8_t* pw = ra.pairs + (size_t)rec * (uint32_t)record_bytes_for(kBmax);   // this lane's two words of pair 0
  ld_stream2_at<0>(pw, r.p[0], r.p[1]);
  ld_stream2_at_if<1 * kPairBytes>(b > 2, pw, r.p[2], r.p[3]);
  ld_stream2_at_if<2 * kPairBytes>(b > 4, pw, r.p[4], r.p[5]);
  ld_stream2_at_if<3 * kPairBytes>(b > 6, pw, r.p[6], r.p[7]);
}

// Truncated codes of this lane's 32 columns for a row of width b (1..8, chosen
// at run time), with one indirect jump: the top plane of the last pair for odd
// b, the full pair for even b, then the full pairs below it in one shared
// sequence. out[j] byte i = top-b bits of column 4j+i, in place, low bits zero;
// mid = the bin midpoint in kBmax-bit units (0 at b = kBmax), fixed by the jump
// target. Widths above kBmax never reach the kernel (the host rejects them).
template <int kBmax>
__device__ __forceinline__ void assemble_row(const RowRegs& r, uint32_t (&out)[8], float& mid) {
  uint32_t T[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) T[j] = 0u;
  switch (r.b) {
    case 8: mid = midpoint<kBmax>(8); merge_pair<3>(r.p[6], r.p[7], T); goto pairs3;
    case 7: mid = midpoint<kBmax>(7); merge_pair_top<3>(r.p[6], r.p[7], T); goto pairs3;
    case 6:
      mid = midpoint<kBmax>(6);
    pairs3:
      merge_pair<2>(r.p[4], r.p[5], T);
      goto pairs2;
    case 5: mid = midpoint<kBmax>(5); merge_pair_top<2>(r.p[4], r.p[5], T); goto pairs2;
    case 4:
      mid = midpoint<kBmax>(4);
    pairs2:
      merge_pair<1>(r.p[2], r.p[3], T);
      goto pairs1;
    case 3: mid = midpoint<kBmax>(3); merge_pair_top<1>(r.p[2], r.p[3], T); goto pairs1;
    case 2:
      mid = midpoint<kBmax>(2);
    pairs1:
      merge_pair<0>(r.p[0], r.p[1], T);
      break;
    default: mid = midpoint<kBmax>(1); merge_pair_top<0>(r.p[0], r.p[1], T); break;   // b == 1
  }
  finish_codes(T, out);
}

// Ask L2 for what one row (k | b << 24) will load: the 2 ceil(b/2) plane lines
// of its record (lane p < 2 ceil(b/2): line p, 128 bytes) and its scale/zero
// words (lane b_max, 32 bytes), one request per lane under a predicate.
__device__ __forceinline__ void prefetch_row_l2(const RowAddr& ra, uint32_t info, int b_max) {
  const uint32_t rec = (info & 0xFFFFFFu) * ra.nt + ra.t;
  const uint32_t lines = ((info >> 24) + 1u) & ~1u;
  const uint8_t* line = ra.line + (size_t)rec * ra.line_mul;
  const uint32_t on = (ra.lane < lines || ra.lane == (uint32_t)b_max) ? 1u : 0u;
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t@p prefetch.global.L2 [%0];\n\t}" ::"l"(line),
               "r"(on));
}

template <int kBmax>
__device__ __forceinline__ void row_fma(const RowRegs& r, float2 (&acc)[16], float& cacc) {
  uint32_t R[8];
  float mid;
  assemble_row<kBmax>(r, R, mid);
  float A;
  row_coef<kBmax>(r.m, r.xh, mid, A, cacc);
  fma_codes(R, A, acc);
}

// ---------------------------------------------------------------------------
// Fused grading (grinqh_select_vmm): CTA r of R grades the channels k = r,
// r + R, r + 2R, ... itself (the class is the number of thresholds |x_k|
// reaches, whatever their order; NaN reaches none) and stages those of nonzero
// width in ascending k as s.u.rows (k | b << 24). Every CTA so gets every R-th
// channel, a random mix of widths as with the list positions of grinqh_vmm, and
// grades only its own K/R channels: no selection kernel, no kernel boundary, no
// channel list and no grading repeated across CTAs. s.width must be filled.
// Returns the number of rows staged (K <= kFusedMaxK = kIdxCap: one pass).
__device__ __forceinline__ int stage_fused(const VmmArgs& a, const uint16_t* __restrict__ xt, VmmSmem& s, int r,
                                           int R) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nt = a.ct.n - 1;
  float th[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) th[q] = (q < nt) ? __ldg(a.thresholds + q) : 0.0f;
  const int nk = (a.K > r) ? (a.K - r + R - 1) / R : 0;
  const uint32_t lt = (1u << lane) - 1u;
  int base = 0;
#pragma unroll 1
  for (int i0 = 0, rnd = 0; i0 < nk; i0 += kThreads, rnd ^= 1) {
    const int i = i0 + tid;
    uint32_t info = 0u;
    bool keep = false;
    if (i < nk) {
      const int k = r + R * i;
      const float ax = fabsf(__half2float(__ushort_as_half(__ldg(xt + k))));
      int c = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) c += (q < nt && ax >= th[q]) ? 1 : 0;
      const int b = s.width[c];
      keep = b > 0;
      info = (uint32_t)k | ((uint32_t)b << 24);
    }
    // ascending k: warp by warp, lane by lane (rounds alternate their count
    // buffer, so one barrier per round suffices)
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) s.wcnt[rnd][warp] = __popc(m);
    __syncthreads();
    int off = base;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
      const int cq = s.wcnt[rnd][q];
      off += (q < warp) ? cq : 0;
      base += cq;
    }
    if (keep) s.u.rows[off + __popc(m & lt)] = info;
  }
  return base;
}


// kBatch: the grid has a token dimension (grinqh_select_vmm_batch): token z
// reads x + z K, has its own set of partials and its own y row. The
// single-vector kernels are compiled without it.
template <bool kFused, int kBmax, bool kBatch>
__global__ void __launch_bounds__(kThreads, 1) vmm_kernel(const VmmArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  VmmSmem& s = *reinterpret_cast<VmmSmem*>(smem_raw);
  const int tid = threadIdx.x, h = tid >> 5, w = tid & 31;   // warp h, word w = lane
  const int t = blockIdx.x, r = blockIdx.y, R = gridDim.y;
  const uint16_t* xv = kBatch ? a.x + (size_t)blockIdx.z * a.K : a.x;   // this CTA's activation vector

  // This CTA takes list positions r + R e (e = 0, 1, ...); the width-0 class,
  // when there is one, is the first class of the list, so its positions are a
  // prefix e < e0 that is skipped. The first channel indices are loaded
  // together with the class offsets (one memory round trip, not two).
  const int nfull = (a.K > r) ? (a.K - r + R - 1) / R : 0;
  constexpr int kPre = 4;
  int pre_idx[kPre];
  pdl_wait();   // the selection (or the thresholds) and x may come from the kernel just before
  if (!kFused) {
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
      const int e = tid + i * kThreads;
      pre_idx[i] = (e < nfull) ? __ldg(a.idx + r + R * e) : 0;
    }
  }
  if (!kFused && tid <= a.ct.n) s.off[tid] = a.offsets[tid];
#pragma unroll
  for (int c = 0; c < 9; ++c)
    if (tid == c && c < a.ct.n) s.width[c] = a.ct.width[c];
  __syncthreads();
  pdl_launch_dependents();

  const int n = a.ct.n;
  const int a0 = kFused ? 0 : ((s.width[0] == 0) ? s.off[1] : 0);   // first position to read
  const int e0 = (a0 > r) ? (a0 - r + R - 1) / R : 0;               // first e at or past a0
  // this CTA's rows: list positions r + R (e0 + q), q = 0 .. nq_total-1
  const int nq_total = kFused ? 0 : nfull - e0;

  float2 acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = make_float2(0.0f, 0.0f);
  float cacc = 0.0f;

  const int nq_fused = kFused ? stage_fused(a, xv, s, r, R) : 0;   // one pass: K <= kFusedMaxK rows fit
  const int passes_total = kFused ? nq_fused : nq_total;
  for (int qb = 0; qb < passes_total; qb += kIdxCap) {
    const int nq = kFused ? nq_fused : min(kIdxCap, nq_total - qb);
    if (!kFused) {
      __syncthreads();
      if (nfull <= kPre * kThreads) {
        // every row of this CTA is in the prefetched indices
#pragma unroll
        for (int i = 0; i < kPre; ++i) {
          const int e = tid + i * kThreads;
          if (e >= e0 && e < nfull) {
            const int pos = r + R * e;
            int j = 0;
            for (int c = 1; c < n; ++c) j += (pos >= s.off[c]) ? 1 : 0;
            s.u.rows[e - e0] = (uint32_t)pre_idx[i] | ((uint32_t)s.width[j] << 24);
          }
        }
      } else {
        for (int e = tid; e < nq; e += kThreads) {
          const int pos = r + R * (e0 + qb + e);
          int j = 0;
          for (int c = 1; c < n; ++c) j += (pos >= s.off[c]) ? 1 : 0;
          s.u.rows[e] = (uint32_t)a.idx[pos] | ((uint32_t)s.width[j] << 24);
        }
      }
    }
    __syncthreads();
    // rows of this warp in the pass: q = h + 16 m, m = 0 .. nrow-1; row m lives
    // in register slot m % kDepth from its loads until its arithmetic
    const int nrow = (nq > h) ? (nq - h + kWarps - 1) / kWarps : 0;
    const RowAddr ra = row_addr(a, t, w);
    RowRegs S[kDepth];
#pragma unroll
    for (int d = 0; d < kDepth; ++d)
      if (d < nrow) load_row<kBmax>(xv, ra, s.u.rows[h + kWarps * d], S[d]);
#pragma unroll 1
    for (int m = kDepth; m < min(nrow, kDepth + kL2Ahead); ++m) prefetch_row_l2(ra, s.u.rows[h + kWarps * m], kBmax);
    int m0 = 0;
    // blocks whose loads and prefetches all exist: no per-row tests
#pragma unroll 1
    for (; m0 + 2 * kDepth + kL2Ahead <= nrow; m0 += kDepth) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int m = m0 + d;
        row_fma<kBmax>(S[d], acc, cacc);
        load_row<kBmax>(xv, ra, s.u.rows[h + kWarps * (m + kDepth)], S[d]);
        // the record prefix of the row kL2Ahead rows further on goes to L2 now,
        // one 128-byte line per lane, so its register loads later hit L2
        prefetch_row_l2(ra, s.u.rows[h + kWarps * (m + kDepth + kL2Ahead)], kBmax);
      }
    }
    // the last blocks, row by row: first the record prefixes of the rows that no
    // block above sent to L2
#pragma unroll 1
    for (int m = m0 + kDepth + kL2Ahead; m < nrow; ++m) prefetch_row_l2(ra, s.u.rows[h + kWarps * m], kBmax);
#pragma unroll 1
    for (; m0 < nrow; m0 += kDepth) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int m = m0 + d;
        if (m < nrow) {
          row_fma<kBmax>(S[d], acc, cacc);
          if (m + kDepth < nrow) load_row<kBmax>(xv, ra, s.u.rows[h + kWarps * (m + kDepth)], S[d]);
        }
      }
    }
  }
  // ---------------- CTA reduction over the 16 warps ----------------
  // Each warp stores its column sums as soon as its own rows are done (the
  // buffer is not shared with the row list), so only the slowest warp's
  // stores and the final sum follow the barrier.
  float* red = s.u.red;
  {
    float* dst = red + h * kRedStride + w;           // slot c*33 + w holds column 32w + c
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dst[(4 * j + 0) * kRedPitch] = fmaf(acc[2 * j].x, 0x1p54f, cacc);
      dst[(4 * j + 2) * kRedPitch] = fmaf(acc[2 * j].y, 0x1p54f, cacc);
      dst[(4 * j + 1) * kRedPitch] = fmaf(acc[2 * j + 1].x, 0x1p54f, cacc);
      dst[(4 * j + 3) * kRedPitch] = fmaf(acc[2 * j + 1].y, 0x1p54f, cacc);
    }
  }
  __syncthreads();
  // partial[r][column], or y itself when there is a single row split; every
  // column of the tile is written, zeros included, so no clearing is needed
  // (a batch's token blockIdx.z: its y row and its set of partials)
  const size_t tok = kBatch ? blockIdx.z : 0;
  float* out = (R == 1) ? a.y + tok * a.N : a.partial + (tok * R + r) * a.n_tiles * kTileN;
  const int limit = (R == 1) ? a.N : a.n_tiles * kTileN;
#pragma unroll
  for (int e = tid; e < kTileN; e += kThreads) {
    // column e of the tile sits at slot (e % 32) * 33 + e / 32 of every warp
    float v = 0.0f;
#pragma unroll
    for (int rl = 0; rl < kWarps; ++rl) v += red[rl * kRedStride + (e % kWords) * kRedPitch + e / kWords];
    const int col = t * kTileN + e;
    if (col < limit) out[col] = v;
  }
}

// y[col] = sum over r of partial[r][col]: 512 threads = 32 columns x 16
// chains; chain c adds r = c, c + 16, ... in ascending order, then the 16 chains
// are added in a fixed order, so the result does not depend on timing. A chain
// issues all its loads (up to kRedLoads) before it adds, so the partials of a
// column arrive in one memory round trip.
constexpr int kRedChains = 16;
constexpr int kRedLoads = 8;   // R <= 128 in one round trip; larger R loops
template <bool kBatch>
__global__ void __launch_bounds__(32 * kRedChains) reduce_partials_kernel(const float* __restrict__ partial, int R,
                                                                         int stride, float* __restrict__ y, int N) {
  __shared__ float s_part[kRedChains][33];
  pdl_launch_dependents();
  pdl_wait();   // the partials come from the VMM kernel just before
  const int lane = threadIdx.x & 31, chain = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;
  if (kBatch) {   // token blockIdx.y of a batch
    partial += (size_t)blockIdx.y * R * stride;
    y += (size_t)blockIdx.y * N;
  }
  float v = 0.0f;
  if (col < N) {
    for (int r0 = chain; r0 < R; r0 += kRedChains * kRedLoads) {
      float p[kRedLoads];
#pragma unroll
      for (int i = 0; i < kRedLoads; ++i) {
        const int r = r0 + kRedChains * i;
        p[i] = (r < R) ? __ldcg(partial + (size_t)r * stride + col) : 0.0f;
      }
#pragma unroll
      for (int i = 0; i < kRedLoads; ++i) v += p[i];
    }
  }
  s_part[chain][lane] = v;
  __syncthreads();
  if (chain == 0 && col < N) {
    float acc = s_part[0][lane];
#pragma unroll
    for (int c = 1; c < kRedChains; ++c) acc += s_part[c][lane];
    y[col] = acc;
  }
}

// ---------------------------------------------------------------------------
// Nested look-up-table codes (grinqh_vmm_lut): the same records of b_max-bit
// codes in plane pairs, read and rebuilt as above, but a code's value is an
// entry of its row's table for the row's width b, w_hat = T_k[2^b + c_b] with
// c_b the code's top b bits (no bin midpoint, no scale or zero point; the
// records' scale/zero words are not read). Tables are binary16 in heap order,
// 2^(b_max+1) entries per row, so width b's 2^b entries are contiguous.
//
// Per row in flight the warp copies the width-b table into shared memory with
// cp.async (no registers), issued with the row's plane loads three rows ahead.
// Before the row's products the warp rewrites it as fp32 values times x_k (an
// exact product of two binary16 values) in a per-warp slot aligned to 1 KB, so
// a code's shared address is the slot address with its low bits replaced by
// 4 c_b: for b <= 6 one shift per register of four codes and one byte-permute
// per code, for b = 7, 8 a shift and a mask per code. Each weight then costs a
// shared load and half of a paired fp32 add.
constexpr int kLutRaw = 256;                        // binary16 entries of the widest table (b = 8)
constexpr int kLutSlot = 1024;                      // bytes of one fp32 table slot

struct __align__(16) LutSmem {
  uint32_t rows[kIdxCap];                         // k | b << 24 of this CTA's rows, one pass
  float red[kWarps * kRedStride];                 // per-warp column sums
  uint16_t raw[kWarps][kDepth][kLutRaw];          // tables as copied, one slot per row in flight
  uint8_t tab[kWarps * kDepth * kLutSlot + kLutSlot];   // x_k-scaled fp32 tables (1 KB-aligned slots)
  int off[10];
  int width[9];
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16_if(bool on, uint32_t dst, const void* src) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %2, 0;\n\t@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}" ::"r"(dst),
      "l"(src), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}
__device__ __forceinline__ void warp_sync_mem() { asm volatile("bar.warp.sync 0xffffffff;" ::: "memory"); }
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// Issue the loads of one row (k | b << 24, b >= 1): x_k, this lane's words of
// plane pairs 0..ceil(b/2)-1, and the row's width-b table into the warp's raw
// slot (entries [0, 16) of the row for b <= 3, which hold widths 1..3, else
// entries [2^b, 2^(b+1)); 16-byte copies, lane l the l-th), as one cp.async
// group. The table buffer holds 2^(kBmax+2) bytes per row, 16-byte aligned.
template <int kBmax>
__device__ __forceinline__ void load_row_lut(const uint16_t* __restrict__ x, const uint8_t* __restrict__ lut,
                                             const RowAddr& ra, uint32_t info, uint32_t raw, int lane,
                                             RowRegs& r) {
  constexpr uint32_t kRowBytes = 1u << (kBmax + 2);
  const uint32_t k = info & 0xFFFFFFu, b = info >> 24;
  const uint32_t rec = k * ra.nt + ra.t;
  r.b = b;
  r.xh = __ldg(x + k);
  const uint8_t* pw = ra.pairs + (size_t)rec * (uint32_t)record_bytes_for(kBmax);
  ld_stream2_at<0>(pw, r.p[0], r.p[1]);
  ld_stream2_at_if<1 * kPairBytes>(b > 2, pw, r.p[2], r.p[3]);
  ld_stream2_at_if<2 * kPairBytes>(b > 4, pw, r.p[4], r.p[5]);
  ld_stream2_at_if<3 * kPairBytes>(b > 6, pw, r.p[6], r.p[7]);
  const uint32_t off = (b <= 3) ? 0u : (2u << b);
  const uint32_t bytes = (b <= 3) ? (kRowBytes < 32u ? kRowBytes : 32u) : (2u << b);
  const uint32_t l16 = 16u * (uint32_t)lane;
  cp_async16_if(l16 < bytes, raw + l16, lut + (size_t)k * kRowBytes + off + l16);
  cp_async_commit();
}

// The products of one row: wait for its table (the kDepth - 1 rows loaded after
// it may still be in flight), scale it by x_k into the fp32 slot, then add the
// looked-up values of this lane's 32 columns. acc[2j] holds columns 4j, 4j+1 and
// acc[2j+1] columns 4j+2, 4j+3 of the lane's 32.
template <int kBmax>
__device__ __forceinline__ void row_lut(const RowRegs& r, uint32_t raw, uint32_t tab, int lane,
                                        float2 (&acc)[16]) {
  cp_async_wait<kDepth - 1>();
  warp_sync_mem();
  const uint32_t b = r.b;
  const float xk = __half2float(__ushort_as_half((unsigned short)r.xh));
  const uint32_t e0 = (b <= 3) ? (1u << b) : 0u;   // width b's first entry in the raw slot
  for (uint32_t c = (uint32_t)lane; c < (1u << b); c += 32u)
    sts_f32(tab + 4u * c, xk * half_bits_to_float(lds_u16(raw + 2u * (e0 + c))));
  warp_sync_mem();
  uint32_t R[8];
  float mid;
  assemble_row<kBmax>(r, R, mid);
  if (b <= 6) {
    // byte i of R >> (6 - b) is 4 c_b of column 4j + i (the bits below a code are zero)
    const uint32_t sh = 6u - b;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t t = R[j] >> sh;
      const float v0 = lds_f32(__byte_perm(t, tab, 0x7650));
      const float v1 = lds_f32(__byte_perm(t, tab, 0x7651));
      const float v2 = lds_f32(__byte_perm(t, tab, 0x7652));
      const float v3 = lds_f32(__byte_perm(t, tab, 0x7653));
      acc[2 * j] = __fadd2_rn(acc[2 * j], make_float2(v0, v1));
      acc[2 * j + 1] = __fadd2_rn(acc[2 * j + 1], make_float2(v2, v3));
    }
  } else {
    const uint32_t mask = ((1u << b) - 1u) << 2;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v0 = lds_f32(((R[j] << (b - 6u)) & mask) | tab);
      const float v1 = lds_f32(((R[j] >> (14u - b)) & mask) | tab);
      const float v2 = lds_f32(((R[j] >> (22u - b)) & mask) | tab);
      const float v3 = lds_f32(((R[j] >> (30u - b)) & mask) | tab);
      acc[2 * j] = __fadd2_rn(acc[2 * j], make_float2(v0, v1));
      acc[2 * j + 1] = __fadd2_rn(acc[2 * j + 1], make_float2(v2, v3));
    }
  }
}

template <int kBmax>
__global__ void __launch_bounds__(kThreads, 1) vmm_lut_kernel(const VmmArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  LutSmem& s = *reinterpret_cast<LutSmem*>(smem_raw);
  const int tid = threadIdx.x, h = tid >> 5, w = tid & 31;
  const int t = blockIdx.x, r = blockIdx.y, R = gridDim.y;
  const uint16_t* xv = a.x;

  // list positions r + R e, the width-0 prefix skipped (as grinqh_vmm)
  const int nfull = (a.K > r) ? (a.K - r + R - 1) / R : 0;
  constexpr int kPre = 4;
  int pre_idx[kPre];
  pdl_wait();
#pragma unroll
  for (int i = 0; i < kPre; ++i) {
    const int e = tid + i * kThreads;
    pre_idx[i] = (e < nfull) ? __ldg(a.idx + r + R * e) : 0;
  }
  if (tid <= a.ct.n) s.off[tid] = a.offsets[tid];
#pragma unroll
  for (int c = 0; c < 9; ++c)
    if (tid == c && c < a.ct.n) s.width[c] = a.ct.width[c];
  __syncthreads();
  pdl_launch_dependents();

  const int n = a.ct.n;
  const int a0 = (s.width[0] == 0) ? s.off[1] : 0;
  const int e0 = (a0 > r) ? (a0 - r + R - 1) / R : 0;
  const int nq_total = nfull - e0;

  float2 acc[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) acc[c] = make_float2(0.0f, 0.0f);

  const uint32_t raw0 = smem_u32(&s.raw[h][0][0]);
  const uint32_t tab0 = ((smem_u32(s.tab) + (kLutSlot - 1u)) & ~(uint32_t)(kLutSlot - 1)) +
                        (uint32_t)h * (kDepth * kLutSlot);
  for (int qb = 0; qb < nq_total; qb += kIdxCap) {
    const int nq = min(kIdxCap, nq_total - qb);
    __syncthreads();
    if (nfull <= kPre * kThreads) {
#pragma unroll
      for (int i = 0; i < kPre; ++i) {
        const int e = tid + i * kThreads;
        if (e >= e0 && e < nfull) {
          const int pos = r + R * e;
          int j = 0;
          for (int c = 1; c < n; ++c) j += (pos >= s.off[c]) ? 1 : 0;
          s.rows[e - e0] = (uint32_t)pre_idx[i] | ((uint32_t)s.width[j] << 24);
        }
      }
    } else {
      for (int e = tid; e < nq; e += kThreads) {
        const int pos = r + R * (e0 + qb + e);
        int j = 0;
        for (int c = 1; c < n; ++c) j += (pos >= s.off[c]) ? 1 : 0;
        s.rows[e] = (uint32_t)a.idx[pos] | ((uint32_t)s.width[j] << 24);
      }
    }
    __syncthreads();
    const int nrow = (nq > h) ? (nq - h + kWarps - 1) / kWarps : 0;
    const RowAddr ra = row_addr(a, t, w);
    RowRegs S[kDepth];
    // one cp.async group per row slot, empty where there is no row, so that the
    // row being multiplied always has exactly kDepth - 1 groups after its own
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      if (d < nrow) load_row_lut<kBmax>(xv, a.lut, ra, s.rows[h + kWarps * d], raw0 + d * 2 * kLutRaw, w, S[d]);
      else cp_async_commit();
    }
#pragma unroll 1
    for (int m = kDepth; m < min(nrow, kDepth + kL2Ahead); ++m) prefetch_row_l2(ra, s.rows[h + kWarps * m], kBmax);
    int m0 = 0;
#pragma unroll 1
    for (; m0 + 2 * kDepth + kL2Ahead <= nrow; m0 += kDepth) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int m = m0 + d;
        row_lut<kBmax>(S[d], raw0 + d * 2 * kLutRaw, tab0 + d * kLutSlot, w, acc);
        load_row_lut<kBmax>(xv, a.lut, ra, s.rows[h + kWarps * (m + kDepth)], raw0 + d * 2 * kLutRaw, w, S[d]);
        prefetch_row_l2(ra, s.rows[h + kWarps * (m + kDepth + kL2Ahead)], kBmax);
      }
    }
#pragma unroll 1
    for (int m = m0 + kDepth + kL2Ahead; m < nrow; ++m) prefetch_row_l2(ra, s.rows[h + kWarps * m], kBmax);
#pragma unroll 1
    for (; m0 < nrow; m0 += kDepth) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int m = m0 + d;
        if (m < nrow) {
          row_lut<kBmax>(S[d], raw0 + d * 2 * kLutRaw, tab0 + d * kLutSlot, w, acc);
          if (m + kDepth < nrow)
            load_row_lut<kBmax>(xv, a.lut, ra, s.rows[h + kWarps * (m + kDepth)], raw0 + d * 2 * kLutRaw, w, S[d]);
          else
            cp_async_commit();
        }
      }
    }
  }
  cp_async_wait<0>();

  // CTA reduction over the 16 warps, as grinqh_vmm
  float* red = s.red;
  {
    float* dst = red + h * kRedStride + w;   // slot c*33 + w holds column 32w + c
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dst[(4 * j + 0) * kRedPitch] = acc[2 * j].x;
      dst[(4 * j + 1) * kRedPitch] = acc[2 * j].y;
      dst[(4 * j + 2) * kRedPitch] = acc[2 * j + 1].x;
      dst[(4 * j + 3) * kRedPitch] = acc[2 * j + 1].y;
    }
  }
  __syncthreads();
  float* out = (R == 1) ? a.y : a.partial + (size_t)r * a.n_tiles * kTileN;
  const int limit = (R == 1) ? a.N : a.n_tiles * kTileN;
#pragma unroll
  for (int e = tid; e < kTileN; e += kThreads) {
    float v = 0.0f;
#pragma unroll
    for (int rl = 0; rl < kWarps; ++rl) v += red[rl * kRedStride + (e % kWords) * kRedPitch + e / kWords];
    const int col = t * kTileN + e;
    if (col < limit) out[col] = v;
  }
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Row splits per column tile: one CTA per SM in total, but at most half the
// SMs for one tile: a layer with one or two column tiles then gives each warp
// a few rows instead of one, and the partial-sum kernel reads half as many
// partials per column (measured faster on 4096 x 1024 layers).
static int row_splits(int n_tiles) {
  const int sms = sm_count();
  const int R = min(sms / 2, sms / n_tiles);
  return R < 1 ? 1 : R;
}

// status word (16 B), then partial[tokens][R][n_tiles * 1024] floats when R > 1
size_t vmm_workspace_bytes_batch(int n_tiles, int tokens) {
  const int R = row_splits(n_tiles);
  return 16 + (R > 1 ? (size_t)tokens * R * n_tiles * kTileN * sizeof(float) : 0);
}

size_t vmm_workspace_bytes(int n_tiles, int /*tile_n*/) { return vmm_workspace_bytes_batch(n_tiles, 1); }

template <int kBmax>
static cudaError_t set_smem_attr() {
  const int smem = (int)sizeof(VmmSmem);
  const cudaFuncAttribute at = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaFuncSetAttribute(vmm_kernel<false, kBmax, false>, at, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(vmm_kernel<true, kBmax, false>, at, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(vmm_kernel<true, kBmax, true>, at, smem);
  return e;
}

template <int kBmax>
static cudaError_t launch_one(const cudaLaunchConfig_t& cfg, const VmmArgs& a, bool fused) {
  if (a.tokens > 1) return cudaLaunchKernelEx(&cfg, vmm_kernel<true, kBmax, true>, a);   // only the fused call batches
  return fused ? cudaLaunchKernelEx(&cfg, vmm_kernel<true, kBmax, false>, a)
               : cudaLaunchKernelEx(&cfg, vmm_kernel<false, kBmax, false>, a);
}

// The kernels' shared-memory limit is raised once per device (with that device
// current); calls from several host threads may race here, so the flag is atomic
// and setting the attribute twice is harmless.
static cudaError_t ensure_smem_attrs() {
  constexpr int kMaxDevices = 64;
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = set_smem_attr<8>();
  if (e == cudaSuccess) e = set_smem_attr<6>();
  if (e == cudaSuccess) e = set_smem_attr<4>();
  if (e == cudaSuccess) e = set_smem_attr<2>();
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
  return e;
}

cudaError_t launch_vmm(const VmmArgs& a, cudaStream_t st, bool fused) {
  const int smem = (int)sizeof(VmmSmem);
  cudaError_t ea = ensure_smem_attrs();
  if (ea != cudaSuccess) return ea;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  const int R = row_splits(a.n_tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_tiles, R, a.tokens > 1 ? a.tokens : 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (a.b_max) {
    case 2: e = launch_one<2>(cfg, a, fused); break;
    case 4: e = launch_one<4>(cfg, a, fused); break;
    case 6: e = launch_one<6>(cfg, a, fused); break;
    case 8: e = launch_one<8>(cfg, a, fused); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || R == 1) return e;

  cudaLaunchConfig_t rc = {};
  rc.gridDim = dim3((a.N + 31) / 32, a.tokens > 1 ? a.tokens : 1, 1);
  rc.blockDim = dim3(32 * kRedChains, 1, 1);
  rc.stream = st;
  rc.attrs = attr;
  rc.numAttrs = 1;
  if (a.tokens > 1)
    return cudaLaunchKernelEx(&rc, reduce_partials_kernel<true>, (const float*)a.partial, R, a.n_tiles * kTileN,
                              a.y, a.N);
  return cudaLaunchKernelEx(&rc, reduce_partials_kernel<false>, (const float*)a.partial, R, a.n_tiles * kTileN, a.y,
                            a.N);
}

// grinqh_vmm_lut: the table kernel, then the partial sums as for grinqh_vmm.
template <int kBmax>
static cudaError_t launch_lut_one(const cudaLaunchConfig_t& cfg, const VmmArgs& a) {
  static_assert(sizeof(LutSmem) + 16 <= 227 * 1024, "table kernel shared memory");
  return cudaLaunchKernelEx(&cfg, vmm_lut_kernel<kBmax>, a);
}

static cudaError_t ensure_lut_smem_attrs() {
  constexpr int kMaxDevices = 64;
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const int smem = (int)sizeof(LutSmem);
  const cudaFuncAttribute at = cudaFuncAttributeMaxDynamicSharedMemorySize;
  e = cudaFuncSetAttribute(vmm_lut_kernel<8>, at, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(vmm_lut_kernel<6>, at, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(vmm_lut_kernel<4>, at, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(vmm_lut_kernel<2>, at, smem);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
  return e;
}

cudaError_t launch_vmm_lut(const VmmArgs& a, cudaStream_t st) {
  cudaError_t e = ensure_lut_smem_attrs();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const int R = row_splits(a.n_tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_tiles, R, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (int)sizeof(LutSmem);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (a.b_max) {
    case 2: e = launch_lut_one<2>(cfg, a); break;
    case 4: e = launch_lut_one<4>(cfg, a); break;
    case 6: e = launch_lut_one<6>(cfg, a); break;
    case 8: e = launch_lut_one<8>(cfg, a); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || R == 1) return e;
  cudaLaunchConfig_t rc = {};
  rc.gridDim = dim3((a.N + 31) / 32, 1, 1);
  rc.blockDim = dim3(32 * kRedChains, 1, 1);
  rc.stream = st;
  rc.attrs = attr;
  rc.numAttrs = 1;
  return cudaLaunchKernelEx(&rc, reduce_partials_kernel<false>, (const float*)a.partial, R, a.n_tiles * kTileN, a.y,
                            a.N);
}

// ---------------------------------------------------------------------------
// Scratch of grinqh_vmm_noalloc: one file-scope device array, shared by every
// call of that entry point on a device. Layout as a caller's workspace: the
// 16-byte status word (zero from module load, like every static device
// variable; this version never sets it), then the partials [R][n_tiles * 1024],
// which every call rewrites completely. Calls that overlap on the GPU race on
// the partials.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB
static __device__ __align__(256) uint8_t g_vmm_scratch[kNoAllocScratchBytes];

size_t vmm_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

int vmm_fused_max_k() { return kFusedMaxK; }

// The scratch's device address in the current device's context. Looked up on
// every call: a host-side query, and a context that was reset and created again
// may have loaded the module (and the array) at another address.
cudaError_t vmm_noalloc_scratch(void** ptr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_vmm_scratch);
  if (e != cudaSuccess) return e;
  *ptr = p;
  return cudaSuccess;
}

}  // namespace grinqh
