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
// halves added in the epilogue. The four K = 16 MMAs of a stage and class go to
// four accumulators (summed at the end), so that no MMA waits for the result of
// the one issued just before it. The second term is a per-token constant of the
// group, added in fp32 at the end. A binary16 overflow (|x m| rounded to binary16
// >= 32768, or a scale of 2^(14 - b_max) or more) sets bit 1 of the status word:
// the launch's Y is then not valid.
//
// One CTA computes one 128-column group (the MMA's M) for up to 32 tokens (the
// MMA's N is twice that, padded to 16 tokens), looping over K in stages of 64
// rows; a step is one stage with up to four active classes (more classes take
// more steps per stage) and owns one slot of a 2-deep shared-memory ring (per
// class 16 KB of codes and 8 KB of activations), so the roles meet once per stage:
//   warp 0      allocates the TMEM columns and, from one lane, issues per step and
//               class four K = 16 MMAs;
//   warps 1..8  read a stage's plane words (three stages ahead), merge each row's
//               codes once, and per class write the masked codes as binary16
//               (the row's exponent byte over c, minus 2^pe 1024: exact) in the
//               MN-major 128-byte-swizzled layout of the A descriptor; then the
//               epilogue;
//   warps 9..16 grade the stage's (token, row) pairs against the thresholds,
//               form the hi/lo parts once, and per class write the masked parts in
//               the K-major 128-byte-swizzled layout of the B descriptor; they also
//               accumulate the per-token constant (Tp / 4 of them: 8 rows a thread).
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
constexpr int kQAcc = 4;                         // accumulators, one per K = 16 step of a stage
constexpr int kQAccCols = 2 * kQMaxTok;          // one accumulator: hi products, then lo products
constexpr int kQTmemCols = kQAcc * kQAccCols;
constexpr int kQRebuildWarps = 8, kQBuildWarps = 8;
constexpr int kQBuildThreads = 32 * kQBuildWarps;
static_assert(kQBuildThreads >= 8 * kQMaxTok, "one 8-row chunk per grading thread");
constexpr int kQThreads = 32 * (1 + kQRebuildWarps + kQBuildWarps);
constexpr int kQAhead = 3;                       // stages a rebuild lane loads ahead

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
  float mid[9];                        // bin midpoint of every class of nonzero width
  uint32_t actmask;                    // bit j: class j has nonzero width
  int n_th;                            // thresholds
  unsigned short thh[8];               // the thresholds rounded up to binary16 (NaN past the last)
  float corr[kQMaxTok];                // per token: sum of x s (mid - z) over this CTA's rows
};

constexpr size_t kQSmem = 1024 + (size_t)kQRing * kQSlot + sizeof(QSync);
static_assert(kQSmem <= 227 * 1024, "batch kernel shared memory");
static_assert(kQMaxTok * kQM * 4 <= kQRing * kQSlot, "the split's accumulator copy fits the ring");

// prmt.b32 in its generic mode: a selector nibble with its top bit set fills the
// result byte with the top bit of the source byte it names (the CUDA intrinsic
// __byte_perm uses only the low three bits of each nibble)
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(0u), "r"(sel));
  return r;
}

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
      bar_init(saddr(&sy.full_b[i]), Tp / 4);   // the grading warps with tokens (8 rows a thread)
      bar_init(saddr(&sy.empty[i]), 1);
    }
    bar_init(saddr(&sy.accum), 1);
    sy.failed = 0u;
    int na = 0;
    uint32_t am = 0u;
    for (int j = 0; j < 9; ++j) {
      const int b = (j < ct.n) ? ct.width[j] : 0;
      sy.width[j] = b;
      sy.mid[j] = (b <= 0 || b >= kBmax) ? 0.0f : (float)(1u << (kBmax - b - 1));
      if (b > 0) {
        sy.act[na++] = j;
        am |= 1u << j;
      }
    }
    sy.n_act = na;
    sy.actmask = am;
    sy.n_th = ct.n - 1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < 8)
    sy.thh[threadIdx.x] = (threadIdx.x < ct.n - 1)
                              ? __half_as_ushort(__float2half_ru(__ldg(thresholds + threadIdx.x)))
                              : (unsigned short)0x7E00u;
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
            mma_f16(tmem + (uint32_t)(kk * kQAccCols), ad0 + oa + kk * (4096 >> 4), bd0 + ob + kk * (32 >> 4),
                    idesc, (u > 0 || ci > 0) ? 1u : 0u);
        }
        mma_commit(saddr(&sy.empty[slot]));
      }
      __syncwarp();
    }
    if (ok && lane == 0) mma_commit(saddr(&sy.accum));   // with no step it arrives at once
    __syncwarp();
  } else if (warp <= kQRebuildWarps) {
    // ---------------- codes: rebuild once per row, mask per class ----------------
    // warp d rebuilds k rows 8 d .. 8 d + 7 of a stage (lane = row + 8 q); lane
    // quarter q owns columns 32 q .. 32 q + 31 of the group, record word 4 sl + q.
    // The 8 lanes of one 128-byte store phase then hold the 8 rows of one swizzle
    // atom at the same column chunk, which the swizzle spreads over all 32 banks.
    const int d = warp - 1, q = lane >> 3;
    const int w = 4 * sl + q;
    const int kl = 8 * d + (lane & 7);
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
    // the masks of the first kQCls active classes (every class when at most four are
    // active) in registers: keep the exponent bytes and the top b bits of every code byte
    uint32_t topc[kQCls];
#pragma unroll
    for (int ci = 0; ci < kQCls; ++ci) {
      const uint32_t b = (ci < n_act) ? (uint32_t)sy.width[sy.act[ci]] : 8u;
      topc[ci] = 0xFF00FF00u | (((0xFFu << (8u - b)) & 0xFFu) * 0x00010001u);
    }
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
        // F[2j], F[2j+1]: the binary16 pairs {2^pe (1024 + c0), 2^pe (1024 + c1)} and
        // {2^pe (1024 + c2), 2^pe (1024 + c3)} of the four codes in R[j]
        uint32_t F[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          F[2 * j] = __byte_perm(R[j], ebx4, 0x5140u);
          F[2 * j + 1] = __byte_perm(R[j], ebx4, 0x7362u);
        }
        if (it + kQAhead < n_k) load_stage(it + kQAhead, buf[i]);
        for (int gi = 0; gi < n_grp && ok; ++gi) {
          const int u = it * n_grp + gi;
          const int slot = u % kQRing;
          ok = bar_wait(saddr(&sy.empty[slot]), ((uint32_t)(u / kQRing) & 1u) ^ 1u);
          if (!ok) break;
          const int ncl = min(kQCls, n_act - gi * kQCls);
#pragma unroll
          for (int ci = 0; ci < kQCls; ++ci) {
          if (ci >= ncl) break;
          uint32_t top = topc[ci];
          if (gi > 0) {
            const uint32_t b = (uint32_t)sy.width[sy.act[gi * kQCls + ci]];
            top = 0xFF00FF00u | (((0xFFu << (8u - b)) & 0xFFu) * 0x00010001u);
          }
          const uint32_t row = a0 + slot * kQSlot + ci * kQABytes + row_off;
          uint32_t h[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t v = F[j] & top;
            const __half2 e = __hsub2(*reinterpret_cast<const __half2*>(&v), c2);
            h[j] = *reinterpret_cast<const uint32_t*>(&e);
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
    // 8 kc .. 8 kc + 7 of token t (at most 32 tokens: one chunk per thread, Tp / 4
    // warps; the others have nothing to do); its x and scale/zero words are loaded
    // one stage ahead. Rows are taken in pairs, as binary16 pairs:
    //   class: the number of thresholds |x| reaches, counted as 1024 + j in
    //     binary16 (HSET2 results added); a binary16 |x| reaches the threshold th
    //     exactly when it reaches th rounded up to binary16;
    //   hi = fp16(x m) and lo = fp16(x m - hi) (one fused multiply-add: x m - hi
    //     is exact in binary32, so it is rounded once, as in two steps);
    //   the per-token constant x s (mid - z) in fp32 (x s exact).
    const int id = threadIdx.x - 32 * (1 + kQRebuildWarps);
    const int nch = Tp * 8;   // a multiple of 32: whole warps
    if (id < nch) {
      const int t = id >> 3, kc = id & 7;
      const bool mine = t < Tc;   // padding tokens stay zero
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
      __half2 th2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) th2[i] = __half2half2(__ushort_as_half(sy.thh[i]));
      const bool few = sy.n_th <= 4;
      const uint32_t actmask = sy.actmask;
      uint32_t jxc[kQCls];   // the first kQCls active classes, one per byte
#pragma unroll
      for (int ci = 0; ci < kQCls; ++ci) jxc[ci] = (ci < n_act) ? (uint32_t)sy.act[ci] * 0x01010101u : 0u;
      __half2 amax = __float2half2_rn(0.0f);
      uint4 xn;
      uint32_t mn[8];
      load_chunk(0, xn, mn);
      for (int it = 0; it < n_k && ok; ++it) {
        const uint4 xv = xn;
        uint32_t mw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mw[e] = mn[e];
        if (it + 1 < n_k) load_chunk(it + 1, xn, mn);
        uint32_t hw[4], lw[4], cnt[4];
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const uint32_t x2b = xw[p];
          const uint32_t s2b = __byte_perm(mw[2 * p], mw[2 * p + 1], 0x5410u);   // scales of rows 2p, 2p+1
          const uint32_t z2b = __byte_perm(mw[2 * p], mw[2 * p + 1], 0x7632u);   // zero points
          const __half2 x2 = *reinterpret_cast<const __half2*>(&x2b);
          const __half2 s2 = *reinterpret_cast<const __half2*>(&s2b);
          const __half2 ax2 = __habs2(x2);
          __half2 c2 = __float2half2_rn(1024.0f);
#pragma unroll
          for (int i = 0; i < 4; ++i) c2 = __hadd2(c2, __hge2(ax2, th2[i]));   // NaN reaches none
          if (!few) {
#pragma unroll
            for (int i = 4; i < 8; ++i) c2 = __hadd2(c2, __hge2(ax2, th2[i]));
          }
          cnt[p] = *reinterpret_cast<const uint32_t*>(&c2);   // low byte of each half: the class
          // m: the scale's significand in [1, 2); s 2^14 (exact) for a subnormal scale
          const uint32_t norm = (s2b & 0x03FF03FFu) | 0x3C003C00u;
          const __half2 sub = __hmul2(s2, __float2half2_rn(16384.0f));
          const uint32_t isn = ((s2b & 0x7C007C00u) + 0x7FFF7FFFu) & 0x80008000u;   // bit 15 of a half: normal
          const uint32_t sel = prmt_sign(isn, 0xBB99u);                        // 0xFFFF where normal
          const uint32_t m2b = (norm & sel) | (*reinterpret_cast<const uint32_t*>(&sub) & ~sel);
          const __half2 m2 = *reinterpret_cast<const __half2*>(&m2b);
          const __half2 hi = __hmul2(x2, m2);
          const __half2 lo = __hfma2(x2, m2, __hneg2(hi));
          amax = __hmax2(amax, __habs2(hi));   // NaN (x NaN, or inf times 0) is passed over
          hw[p] = *reinterpret_cast<const uint32_t*>(&hi);
          lw[p] = *reinterpret_cast<const uint32_t*>(&lo);
#pragma unroll
          for (int l = 0; l < 2; ++l) {
            const uint32_t j = (cnt[p] >> (16 * l)) & 0xFu;
            const float x = half_bits_to_float(x2b >> (16 * l));
            const float sv = half_bits_to_float(s2b >> (16 * l));
            const float z = half_bits_to_float(z2b >> (16 * l));
            if ((actmask >> j) & 1u) corr = fmaf(x * sv, sy.mid[j] - z, corr);   // x s exact: two 11-bit significands
          }
        }
        // the class of rows 0..3 and 4..7, one byte each
        const uint32_t cb0 = __byte_perm(cnt[0], cnt[1], 0x6420u), cb1 = __byte_perm(cnt[2], cnt[3], 0x6420u);
        for (int gi = 0; gi < n_grp && ok; ++gi) {
          const int u = it * n_grp + gi;
          const int slot = u % kQRing;
          ok = bar_wait(saddr(&sy.empty[slot]), ((uint32_t)(u / kQRing) & 1u) ^ 1u);
          if (!ok) break;
          const int ncl = min(kQCls, n_act - gi * kQCls);
          // row t (hi) and row Tp + t (lo) of the K-major tile: 8-row groups 1 KB
          // apart, 128 bytes per row, 16-byte chunk kc stored at chunk index kc ^ (row
          // % 8); Tp is a multiple of 16, so row Tp + t sits Tp * 128 bytes after row t
          const uint32_t off = (uint32_t)((t >> 3) * 1024 + (t & 7) * 128) + ((uint32_t)(kc ^ (t & 7)) << 4);
          const uint32_t lo_off = (uint32_t)Tp * 128u;
#pragma unroll
          for (int ci = 0; ci < kQCls; ++ci) {
            if (ci >= ncl) break;
            const uint32_t jx = (gi == 0) ? jxc[ci] : (uint32_t)sy.act[gi * kQCls + ci] * 0x01010101u;
            const uint32_t sb = a0 + slot * kQSlot + kQCls * kQABytes + ci * kQBBytes;
            // bit 7 of a byte: that row's class differs (bytes are at most 15, so
            // adding 0x7F carries into no other byte)
            const uint32_t d0 = ((cb0 ^ jx) + 0x7F7F7F7Fu) & 0x80808080u;
            const uint32_t d1 = ((cb1 ^ jx) + 0x7F7F7F7Fu) & 0x80808080u;
            // per half: 0xFFFF where the row's class differs (the byte's top bit replicated)
            const uint32_t k0m = prmt_sign(d0, 0x9988u), k1m = prmt_sign(d0, 0xBBAAu);
            const uint32_t k2m = prmt_sign(d1, 0x9988u), k3m = prmt_sign(d1, 0xBBAAu);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + off), "r"(hw[0] & ~k0m),
                         "r"(hw[1] & ~k1m), "r"(hw[2] & ~k2m), "r"(hw[3] & ~k3m)
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + lo_off + off), "r"(lw[0] & ~k0m),
                         "r"(lw[1] & ~k1m), "r"(lw[2] & ~k2m), "r"(lw[3] & ~k3m)
                         : "memory");
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) bar_arrive(saddr(&sy.full_b[slot]));
        }
      }
      if (__hge(__hmax(__low2half(amax), __high2half(amax)), __float2half_rn(32768.0f))) bad = true;
      // per-token constant: the 8 threads of a token are 8 consecutive lanes
      float v = corr;
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      if (kc == 0) sy.corr[t] = v;
    }
  }
  if (!ok) atomicOr(&sy.failed, 1u);
  if (bad) atomicOr(&sy.failed, 2u);
  tc_before();
  __syncthreads();
  tc_after();
  ok = ok && (sy.failed & 1u) == 0u;

  // ---------------- epilogue ----------------
  // warps 1..4 read TMEM lane quarter (warp % 4): lane i = column n0 + 32 (warp % 4) + i;
  // in accumulator a (columns 64 a ..), column t holds token t's hi product and
  // column Tp + t its lo product; y = the sum of all eight + the token's constant
  float* dump = reinterpret_cast<float*>(q_smem + (a0 - raw));   // [token][column] for the cluster sum
  if (warp >= 1 && warp <= 4) {
    const bool acc_ok = (sy.failed & 1u) == 0u && bar_wait(saddr(&sy.accum), 0u);
    tc_after();
    const int qq = warp & 3;
    const int n = n0 + 32 * qq + lane;
    for (int c16 = 0; c16 < Tp; c16 += 16) {
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
      if (n_act > 0 && n_k > 0) {
#pragma unroll
        for (int part = 0; part < 2 * kQAcc; ++part) {   // accumulator part / 2, hi (even) or lo (odd) half
          uint32_t v[16];
          const uint32_t ta = tmem + ((uint32_t)(32 * qq) << 16) + (uint32_t)((part >> 1) * kQAccCols) +
                              (uint32_t)((part & 1) * Tp + c16);
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
              "%14, %15}, [%16];"
              : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
              : "r"(ta));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] += __uint_as_float(v[i]);
        }
      }   // else no class of nonzero width: only the constant
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = c16 + i;
        const float yv = acc[i] + sy.corr[t < kQMaxTok ? t : 0];
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
