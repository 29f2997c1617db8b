// Graded product for a batch of tokens on the 5th-generation tensor cores
// (sm_100a): Y[t][n] = sum_k x_tk w_hat^(b_tk)[k][n], every token graded from
// its own |x| (Section 3.1) and every row rebuilt at that token's width
// (Section 3.3), as at batch one, but with each row's planes read and merged
// once for all tokens of the launch.
//
// The product is split by width class. With code_b = c_b 2^(b_max-b) + mid_b,
// w_hat = s (code_b - z) and q8 the row's code in the 8-bit frame (plane p at bit
// 7-p), c_b 2^(b_max-b) = 2^(b_max-8) (q8 & top_b), top_b the mask of the top b
// bits. Write the row's scale as s = m 2^(e-15), m its binary16 significand in
// [1, 2) and e its exponent field (for a subnormal s, e = 1 and m = s 2^14). For
// one 128-column group (one scale per row) and class j of width b_j:
//   Y[t][n] += sum_{k: class(t,k) = j} (x_tk m_k) ((q8_kn & top_bj) 2^(e_k-23+b_max))
//            + sum_{k: class(t,k) = j} x_tk s_k (mid_bj - z_k).
// The first term is an MMA per class: A = the codes masked to the class width
// times a power of two, exact in binary16; B = x m in two binary16 parts (hi =
// fp16(v), lo = fp16(v - hi), about 22 significant bits together, near |x| in
// magnitude), zero where the token's class differs, the hi parts of the tokens in
// B's first Tp rows and the lo parts in the next Tp, so that one MMA of N = 2 Tp
// fetches the A tile once for both; fp32 accumulation in tensor memory, the two
// halves added in the epilogue. The second term is a per-token constant of the group, added in fp32 at
// the end. A binary16 overflow (|x m| >= 32768, or a scale of 2^(14 - b_max) or
// more) sets bit 1 of the status word: the launch's Y is then not valid.
//
// One CTA computes one 128-column group (the MMA's M) for up to 32 tokens (the
// MMA's N is twice that, padded to 16 tokens), looping over K in stages of 64
// rows; a step is one stage with up to four active classes (more classes take
// more steps per stage) and owns one slot of a 2-deep shared-memory ring (per
// class 16 KB of codes and 8 KB of activations), so the roles meet once per stage:
//   warp 0      allocates the TMEM columns and, from one lane, issues per step and
//               class four K = 16 MMAs;
//   warps 1..8  read a stage's plane words (two stages ahead), merge each row's
//               codes once, and per class write the masked codes as binary16
//               (the row's exponent byte over c, minus 2^pe 1024: exact) in the
//               MN-major 128-byte-swizzled layout of the A descriptor; then the
//               epilogue;
//   warps 9..16 grade the stage's (token, row) pairs against the thresholds,
//               form the hi/lo parts once, and per class write the masked parts in
//               the K-major 128-byte-swizzled layout of the B descriptor; they also
//               accumulate the per-token constant.
// Small grids split K over a cluster of 2, 4 or 8 CTAs that add their
// accumulators through distributed shared memory in rank order (deterministic).
// Every mbarrier wait is bounded by the global timer; one that gives up sets bit
// 0 of the status word.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace grinqh {
namespace {

constexpr int kQM = 128;                         // output columns per CTA: one group (MMA M)
constexpr int kQK = 64;                          // k rows per stage
constexpr int kQMaxTok = 32;                     // tokens per CTA (MMA N, padded to 16)
constexpr int kQRing = 2;                        // ring slots, one per step
constexpr int kQCls = 4;                         // classes per step
constexpr int kQABytes = kQM * kQK * 2;          // 16 KB: one class's codes
constexpr int kQBBytes = 2 * kQMaxTok * kQK * 2; // 8 KB: one class's hi and lo activations
constexpr int kQSlot = kQCls * (kQABytes + kQBBytes);   // 96 KB: codes of 4 classes, then activations
constexpr int kQTmemCols = 2 * kQMaxTok;         // accumulator: hi products, then lo products
constexpr int kQRebuildWarps = 8, kQBuildWarps = 8;
constexpr int kQBuildThreads = 32 * kQBuildWarps;
static_assert(kQBuildThreads >= 8 * kQMaxTok, "one 8-row chunk per grading thread");
constexpr int kQThreads = 32 * (1 + kQRebuildWarps + kQBuildWarps);
constexpr int kQAhead = 2;                       // stages a rebuild lane loads ahead

struct QSync {
  unsigned long long full_a[kQRing];   // one arrival per rebuild warp
  unsigned long long full_b[kQRing];   // one arrival per grading warp
  unsigned long long empty[kQRing];    // the MMAs that read the slot have completed
  unsigned long long accum;            // every MMA of the CTA has completed
  uint32_t tmem;
  uint32_t failed;
  int n_act;                           // classes of nonzero width
  int act[9];                          // their class indices
  int width[9];                        // width of every class
  float th[8];                         // the thresholds
  float corr[kQMaxTok];                // per token: sum of x s (mid - z) over this CTA's rows
};

constexpr size_t kQSmem = 1024 + (size_t)kQRing * kQSlot + sizeof(QSync);
static_assert(kQSmem <= 227 * 1024, "batch kernel shared memory");
static_assert(kQMaxTok * kQM * 4 <= kQRing * kQSlot, "the split's accumulator copy fits the ring");

struct QWords {
  uint32_t p[8];
  uint32_t m;   // the row's scale | zero word of this CTA's group
};

template <int kBmax>
__device__ __forceinline__ void q_load_words(const uint8_t* __restrict__ planes, const uint8_t* __restrict__ meta,
                                             int w, QWords& v) {
  v.m = __ldg(reinterpret_cast<const uint32_t*>(meta) + (w >> 2));
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    if (2 * s < kBmax) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(planes + s * kPairBytes) + w);
      v.p[2 * s] = u.x;
      v.p[2 * s + 1] = u.y;
    } else {
      v.p[2 * s] = v.p[2 * s + 1] = 0u;
    }
  }
}

template <int kBmax, int kSplit>
__global__ void __launch_bounds__(kQThreads, 1)
    batch_tc_kernel(const uint8_t* __restrict__ packed, size_t meta_offset, const uint16_t* __restrict__ X, int T,
                    int K, int N, int n_tiles, const float* __restrict__ thresholds, ClassTable ct,
                    float* __restrict__ Y, uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t q_smem[];
  const uint32_t raw = saddr(q_smem);
  const uint32_t a0 = (raw + 1023u) & ~1023u;   // 1 KB-aligned ring (swizzle atoms)
  QSync& sy = *reinterpret_cast<QSync*>(q_smem + (a0 - raw) + kQRing * kQSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kQM;              // this CTA's group
  const int tb = blockIdx.y * kQMaxTok;         // first token of this CTA
  const int Tc = min(kQMaxTok, T - tb);         // tokens of this CTA
  const int Tp = (Tc + 15) & ~15;               // MMA N
  X += (size_t)tb * K;
  Y += (size_t)tb * N;
  const int n_k_all = (K + kQK - 1) / kQK;
  const int rank = (kSplit > 1) ? (int)blockIdx.z : 0;
  const int ks0 = (int)(((long long)n_k_all * rank) / kSplit);
  const int n_k = (int)(((long long)n_k_all * (rank + 1)) / kSplit) - ks0;
  const int t_rec = n0 / kTileN, sl = (n0 % kTileN) / kQM;   // record tile and group within it

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQRing; ++i) {
      bar_init(saddr(&sy.full_a[i]), kQRebuildWarps);
      bar_init(saddr(&sy.full_b[i]), kQBuildWarps);
      bar_init(saddr(&sy.empty[i]), 1);
    }
    bar_init(saddr(&sy.accum), 1);
    sy.failed = 0u;
    int na = 0;
    for (int j = 0; j < ct.n; ++j) {
      sy.width[j] = ct.width[j];
      if (ct.width[j] > 0) sy.act[na++] = j;
    }
    sy.n_act = na;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < 8) sy.th[threadIdx.x] = (threadIdx.x < ct.n - 1) ? __ldg(thresholds + threadIdx.x) : 0.0f;
  if (threadIdx.x < kQMaxTok) sy.corr[threadIdx.x] = 0.0f;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&sy.tmem)),
                 "r"(kQTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = sy.tmem;
  const int n_act = sy.n_act;
  const int n_grp = (n_act + kQCls - 1) / kQCls;   // steps per stage
  const int steps = n_k * n_grp;
  bool ok = true;
  bool bad = false;   // a value outside the binary16 range of the operands

  if (warp == 0) {
    // ---------------- MMA issue ----------------
    // kind::f16, D fp32, A (codes) MN-major, B (activations) K-major, M = 128, N = 2 Tp
    const uint32_t idesc = (1u << 4) | (1u << 15) | ((uint32_t)(2 * Tp >> 3) << 17) | ((uint32_t)(kQM >> 4) << 24);
    // descriptors of slot 0, class 0, K step 0; the others differ in the start
    // address field only (bits 0..13, address / 16; no carry out of it: the ring
    // ends below 256 KB)
    const uint64_t ad0 = smem_desc(a0, 1024, 2048);
    const uint64_t bd0 = smem_desc(a0 + kQCls * kQABytes, 16, 1024);
    for (int u = 0; u < steps && ok; ++u) {
      const int slot = u % kQRing;
      const uint32_t ph = (uint32_t)(u / kQRing) & 1u;
      ok = bar_wait(saddr(&sy.full_a[slot]), ph) && bar_wait(saddr(&sy.full_b[slot]), ph);
      tc_after();
      if (ok && lane == 0) {
        const int ncl = min(kQCls, n_act - (u % n_grp) * kQCls);   // classes of this step
        for (int ci = 0; ci < ncl; ++ci) {
          const uint32_t oa = (uint32_t)(slot * kQSlot + ci * kQABytes) >> 4;
          const uint32_t ob = (uint32_t)(slot * kQSlot + ci * kQBBytes) >> 4;
#pragma unroll
          for (int kk = 0; kk < kQK / 16; ++kk)
            mma_f16(tmem, ad0 + oa + kk * (4096 >> 4), bd0 + ob + kk * (32 >> 4), idesc,
                    (u > 0 || ci > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(saddr(&sy.empty[slot]));
      }
      __syncwarp();
    }
    if (ok && lane == 0) mma_commit(saddr(&sy.accum));   // with no step it arrives at once
    __syncwarp();
  } else if (warp <= kQRebuildWarps) {
    // ---------------- codes: rebuild once per row, mask per class ----------------
    // warp d rebuilds k rows 8 d .. 8 d + 7 of a stage (lane = 4 row + q); lane
    // quarter q owns columns 32 q .. 32 q + 31 of the group, record word 4 sl + q
    const int d = warp - 1, q = lane & 3;
    const int w = 4 * sl + q;
    const int kl = 8 * d + (lane >> 2);
    const size_t rbytes = (size_t)record_bytes_for(kBmax);
    const uint32_t r8 = (uint32_t)(kl & 7);
    const uint32_t row_off = (uint32_t)((2 * (kl >> 3) + (q >> 1)) * 1024) + r8 * 128u;
    auto load_stage = [&](int it, QWords& v) {
      const int k = (ks0 + it) * kQK + kl;
      if (k < K) {
        const size_t rec = (size_t)k * n_tiles + t_rec;
        q_load_words<kBmax>(packed + rec * rbytes, packed + meta_offset + rec * kMetaBytes, w, v);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v.p[j] = 0u;
        v.m = 0u;
      }
    };
    QWords buf[kQAhead];
#pragma unroll
    for (int i = 0; i < kQAhead; ++i)
      if (i < n_k) load_stage(i, buf[i]);
    for (int i0 = 0; i0 < n_k && ok; i0 += kQAhead) {
#pragma unroll
      for (int i = 0; i < kQAhead; ++i) {
        const int it = i0 + i;
        if (it >= n_k || !ok) break;
        uint32_t R[8];
        assemble<kBmax>(buf[i].p, R);   // byte i of R[j]: the code of column 4j+i in the 8-bit frame
        // the codes' factor 2^pe, pe = e - 23 + b_max, e = max(1, the scale's exponent
        // field): a code c becomes the binary16 with exponent field pe + 25 and
        // mantissa c, i.e. 2^pe (1024 + c), minus 2^pe 1024 (same exponent: exact)
        const int es = max(1, (int)((buf[i].m >> 10) & 31u));
        const int pe = es - 23 + kBmax;
        if (pe > 5 && buf[i].m != 0u) bad = true;   // exponent field above 30: out of binary16 range
        const uint32_t eb = ((uint32_t)(pe + 25) & 31u) << 2;   // the binary16's high byte
        const uint32_t ebx4 = eb * 0x01010101u;
        const uint32_t cw = ((uint32_t)(pe + 25) & 31u) << 10;   // 2^pe 1024
        const uint32_t cw2 = cw * 0x10001u;
        const __half2 c2 = *reinterpret_cast<const __half2*>(&cw2);
        if (it + kQAhead < n_k) load_stage(it + kQAhead, buf[i]);
        for (int gi = 0; gi < n_grp && ok; ++gi) {
          const int u = it * n_grp + gi;
          const int slot = u % kQRing;
          ok = bar_wait(saddr(&sy.empty[slot]), ((uint32_t)(u / kQRing) & 1u) ^ 1u);
          if (!ok) break;
          const int ncl = min(kQCls, n_act - gi * kQCls);
          for (int ci = 0; ci < ncl; ++ci) {
          const uint32_t b = (uint32_t)sy.width[sy.act[gi * kQCls + ci]];
          const uint32_t top = ((0xFFu << (8u - b)) & 0xFFu) * 0x01010101u;
          const uint32_t row = a0 + slot * kQSlot + ci * kQABytes + row_off;
          uint32_t h[16];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t v = R[j] & top;
            const uint32_t lo = __byte_perm(v, ebx4, 0x5140u);   // {2^pe (1024 + c0), 2^pe (1024 + c1)}
            const uint32_t hi = __byte_perm(v, ebx4, 0x7362u);   // {2^pe (1024 + c2), 2^pe (1024 + c3)}
            const __half2 e0 = __hsub2(*reinterpret_cast<const __half2*>(&lo), c2);
            const __half2 e1 = __hsub2(*reinterpret_cast<const __half2*>(&hi), c2);
            h[2 * j] = *reinterpret_cast<const uint32_t*>(&e0);
            h[2 * j + 1] = *reinterpret_cast<const uint32_t*>(&e1);
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint32_t chunk = ((uint32_t)(4 * (q & 1) + cc)) ^ r8;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + chunk * 16u), "r"(h[4 * cc]),
                         "r"(h[4 * cc + 1]), "r"(h[4 * cc + 2]), "r"(h[4 * cc + 3])
                         : "memory");
          }
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) bar_arrive(saddr(&sy.full_a[slot]));
        }
      }
    }
  } else {
    // ---------------- activations: grade once per stage, mask per class ----------------
    // thread i takes the 8-row chunk i of a stage: chunk id = 8 t + kc is rows
    // 8 kc .. 8 kc + 7 of token t (at most 32 tokens: one chunk per thread); its x
    // and scale/zero words are loaded one stage ahead
    const int id = threadIdx.x - 32 * (1 + kQRebuildWarps);
    const int nch = Tp * 8;
    const int nth = ct.n - 1;   // thresholds
    const int t = id >> 3, kc = id & 7;
    const bool mine = id < nch && t < Tc;   // padding tokens stay zero
    float corr = 0.0f;
    auto load_chunk = [&](int it, uint4& xv, uint32_t (&mw)[8]) {
      const int k0 = (ks0 + it) * kQK + 8 * kc;
      if (mine && k0 < K) {
        xv = __ldg(reinterpret_cast<const uint4*>(X + (size_t)t * K + k0));
#pragma unroll
        for (int e = 0; e < 8; ++e)
          mw[e] = __ldg(reinterpret_cast<const uint32_t*>(packed + meta_offset +
                                                           ((size_t)(k0 + e) * n_tiles + t_rec) * kMetaBytes + 4 * sl));
      } else {
        xv = make_uint4(0u, 0u, 0u, 0u);   // rows past K, padding tokens: x = 0 (class 0, no term)
#pragma unroll
        for (int e = 0; e < 8; ++e) mw[e] = 0u;
      }
    };
    float th[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) th[i] = (i < nth) ? sy.th[i] : __int_as_float(0x7fc00000);   // NaN: no |x| reaches it
    uint4 xn;
    uint32_t mn[8];
    load_chunk(0, xn, mn);
    for (int it = 0; it < n_k && ok; ++it) {
      const uint4 xv = xn;
      uint32_t mw[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mw[e] = mn[e];
      if (it + 1 < n_k) load_chunk(it + 1, xn, mn);
      // hi and lo parts of x m as 4 + 4 half pairs, and the 8 classes, one nibble each
      uint32_t hw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u}, cls = 0u;
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t m = mw[e];
        const float s = half_bits_to_float(m), z = half_bits_to_float(m >> 16);
        const float x = half_bits_to_float((e & 1) ? (xw[e >> 1] >> 16) : xw[e >> 1]);
        const float ax = fabsf(x);
        int j = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) j += (ax >= th[i]) ? 1 : 0;   // NaN reaches none
        const int b = sy.width[j];
        const float xs = x * s;                       // exact: two 11-bit significands
        // m: the scale's significand in [1, 2) (s 2^14 for a subnormal scale)
        const uint32_t sbits = m & 0xFFFFu;
        const float mm = (((sbits >> 10) & 31u) != 0u)
                             ? __half2float(__ushort_as_half((unsigned short)((sbits & 0x3FFu) | 0x3C00u)))
                             : s * 16384.0f;
        const float v = x * mm;                       // exact
        if (fabsf(v) >= 32768.0f) bad = true;
        const __half vh = __float2half_rn(v);
        const __half vl = __float2half_rn(v - __half2float(vh));
        const uint32_t hb = __half_as_ushort(vh), lb = __half_as_ushort(vl);
        hw[e >> 1] |= (e & 1) ? (hb << 16) : hb;
        lw[e >> 1] |= (e & 1) ? (lb << 16) : lb;
        cls |= (uint32_t)j << (4 * e);
        if (b > 0) {
          const float mid = (b >= kBmax) ? 0.0f : (float)(1u << (kBmax - b - 1));
          corr = fmaf(xs, mid - z, corr);
        }
      }
      for (int gi = 0; gi < n_grp && ok; ++gi) {
        const int u = it * n_grp + gi;
        const int slot = u % kQRing;
        ok = bar_wait(saddr(&sy.empty[slot]), ((uint32_t)(u / kQRing) & 1u) ^ 1u);
        if (!ok) break;
        const int ncl = min(kQCls, n_act - gi * kQCls);
        if (id < nch) {
          // row t (hi) and row Tp + t (lo) of the K-major tile: 8-row groups 1 KB
          // apart, 128 bytes per row, 16-byte chunk kc stored at chunk index kc ^ (row
          // % 8); Tp is a multiple of 16, so row Tp + t sits Tp * 128 bytes after row t
          const uint32_t off = (uint32_t)((t >> 3) * 1024 + (t & 7) * 128) + ((uint32_t)(kc ^ (t & 7)) << 4);
          const uint32_t lo_off = (uint32_t)Tp * 128u;
          for (int ci = 0; ci < ncl; ++ci) {
            const uint32_t jc = (uint32_t)sy.act[gi * kQCls + ci];
            const uint32_t sb = a0 + slot * kQSlot + kQCls * kQABytes + ci * kQBBytes;
            uint32_t mh[4], ml[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const uint32_t m0 = (((cls >> (8 * p)) & 0xFu) == jc) ? 0x0000FFFFu : 0u;
              const uint32_t m1 = (((cls >> (8 * p + 4)) & 0xFu) == jc) ? 0xFFFF0000u : 0u;
              mh[p] = hw[p] & (m0 | m1);
              ml[p] = lw[p] & (m0 | m1);
            }
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + off), "r"(mh[0]), "r"(mh[1]),
                         "r"(mh[2]), "r"(mh[3])
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + lo_off + off), "r"(ml[0]),
                         "r"(ml[1]), "r"(ml[2]), "r"(ml[3])
                         : "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(saddr(&sy.full_b[slot]));
      }
    }
    // per-token constant: the 8 threads of a token are 8 consecutive lanes
    float v = corr;
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (kc == 0 && id < nch) sy.corr[t] = v;
  }
  if (!ok) atomicOr(&sy.failed, 1u);
  if (bad) atomicOr(&sy.failed, 2u);
  tc_before();
  __syncthreads();
  tc_after();
  ok = ok && (sy.failed & 1u) == 0u;

  // ---------------- epilogue ----------------
  // warps 1..4 read TMEM lane quarter (warp % 4): lane i = column n0 + 32 (warp % 4) + i,
  // TMEM column t = token t's hi product, column Tp + t its lo product; y = both +
  // the token's constant
  float* dump = reinterpret_cast<float*>(q_smem + (a0 - raw));   // [token][column] for the cluster sum
  if (warp >= 1 && warp <= 4) {
    const bool acc_ok = (sy.failed & 1u) == 0u && bar_wait(saddr(&sy.accum), 0u);
    tc_after();
    const int qq = warp & 3;
    const int n = n0 + 32 * qq + lane;
    for (int c16 = 0; c16 < Tp; c16 += 16) {
      uint32_t v[16], w[16];
      if (n_act > 0 && n_k > 0) {
        const uint32_t ta = tmem + ((uint32_t)(32 * qq) << 16) + (uint32_t)c16;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(ta));
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15}, [%16];"
            : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7]),
              "=r"(w[8]), "=r"(w[9]), "=r"(w[10]), "=r"(w[11]), "=r"(w[12]), "=r"(w[13]), "=r"(w[14]), "=r"(w[15])
            : "r"(ta + (uint32_t)Tp));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = w[i] = 0u;   // no class of nonzero width: only the constant
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = c16 + i;
        const float yv = (__uint_as_float(v[i]) + __uint_as_float(w[i])) + sy.corr[t < kQMaxTok ? t : 0];
        if (kSplit == 1) {
          if (t < Tc && n < N && acc_ok) Y[(size_t)t * N + n] = yv;
        } else {
          dump[t * kQM + 32 * qq + lane] = yv;
        }
      }
    }
    if (!acc_ok && lane == 0) atomicOr(&sy.failed, 1u);
  }
  if (kSplit > 1) {
    __syncthreads();
    cluster_sync_all();
    // rank r adds its share of the tokens over the ranks' copies in rank order
    const int per = (Tp + kSplit - 1) / kSplit;
    const int ta = rank * per, tz = min(Tp, ta + per);
    for (int e = threadIdx.x; e < (tz - ta) * kQM; e += kQThreads) {
      const int t = ta + e / kQM, c = e % kQM;
      const uint32_t off = a0 + (uint32_t)(t * kQM + c) * 4u;
      float v = 0.0f;
#pragma unroll
      for (int r = 0; r < kSplit; ++r) v += ld_dsmem_f32(off, (uint32_t)r);
      const int n = n0 + c;
      if (t < Tc && n < N) Y[(size_t)t * N + n] = v;
    }
    cluster_sync_all();
  }
  tc_before();
  __syncthreads();
  if (threadIdx.x == 0 && sy.failed != 0u) atomicOr(status, sy.failed);
  if (warp == 0) {
    tc_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kQTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t launch_batch_tc(const uint16_t* X, int T, const void* packed, int K, int N, int n_tiles, int b_max,
                            const float* thresholds, const ClassTable& ct, float* Y, uint32_t* status,
                            cudaStream_t st) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms < 1) sms = 1;
  const long long groups = (N + kQM - 1) / kQM;
  const long long chunks = (T + kQMaxTok - 1) / kQMaxTok;
  const int n_k_all = (K + kQK - 1) / kQK;
  // a K split over a cluster when the grid of groups x token chunks is small
  int split = 1;
  for (int sp = 8; sp >= 2; sp /= 2)
    if (sp * groups * chunks <= sms && n_k_all >= sp) {
      split = sp;
      break;
    }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)groups, (unsigned)chunks, (unsigned)split);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = kQSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)split;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const size_t meta_offset = meta_offset_for(K, n_tiles, b_max);
  cudaError_t e;
#define GRINQH_BQ_LAUNCH(B, S)                                                                                 \
  e = cudaFuncSetAttribute(batch_tc_kernel<B, S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQSmem);   \
  if (e != cudaSuccess) return e;                                                                              \
  e = cudaLaunchKernelEx(&cfg, batch_tc_kernel<B, S>, (const uint8_t*)packed, meta_offset, X, T, K, N, n_tiles, \
                         thresholds, ct, Y, status);
#define GRINQH_BQ_CASE(B)                      \
  case B:                                      \
    switch (split) {                           \
      case 8: GRINQH_BQ_LAUNCH(B, 8) break;    \
      case 4: GRINQH_BQ_LAUNCH(B, 4) break;    \
      case 2: GRINQH_BQ_LAUNCH(B, 2) break;    \
      default: GRINQH_BQ_LAUNCH(B, 1) break;   \
    }                                          \
    break;
  switch (b_max) {
    GRINQH_BQ_CASE(2)
    GRINQH_BQ_CASE(4)
    GRINQH_BQ_CASE(6)
    GRINQH_BQ_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef GRINQH_BQ_CASE
#undef GRINQH_BQ_LAUNCH
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace grinqh
