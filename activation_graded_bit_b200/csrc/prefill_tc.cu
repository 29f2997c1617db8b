// Fused prefill product on the 5th-generation tensor cores (sm_100a):
// Y[T][N] = X[T][K] . W_hat[K][N], with W_hat rebuilt from the packed bit planes
// straight into the MMA's shared-memory operand tiles (no binary16 copy of the
// weights in HBM).
//
// Paper: "GRINQH" Section 4, "Prefill vs. Decoding Evaluation": prefill takes
// every weight at its full b_max precision and runs a dense matrix-matrix
// product; Section 5 credits efficient unpacking fused with the product for the
// prefill speed. The operand values are those of grinqh_dequant: w_hat =
// fp16_rne(s * (q - z)) per (row k, 128-column group), q the b_max-bit code.
//
// One CTA computes a tile of 128 output columns (the MMA's M, from W_hat) by 256
// tokens (the MMA's N, from X), or by 512 tokens as two 256-token halves that share
// each rebuilt weight tile (when the grid of such CTAs takes fewer waves), with fp32
// accumulators in tensor memory (256 or 512 columns), looping over K in stages of
// 64 rows held in a 4-deep (256 tokens) or 2-deep (512 tokens) shared-memory ring:
//   warp 0      X tiles by TMA (no multicast): 256 tokens x 64 k per half, K-major,
//               128-byte swizzle, one mbarrier transaction per stage;
//   warp 1      allocates the TMEM columns and, from one lane, issues the four
//               kind::f16 MMAs (K = 16 each) of a stage per token half once both
//               operand tiles are full, then commits to the stage's "empty" barrier;
//   warps 2..9  rebuild the stage's 64 x 128 weight tile, 8 rows per warp: 4 lanes
//               per row, each lane the 32 columns of one record word, written as
//               binary16 in the MN-major 128-byte-swizzled layout the A descriptor
//               names; a lane loads a stage's words three stages before it fills
//               it. Codes become binary16 without an integer
//               conversion: a byte-permute puts code c under the exponent of 1024
//               (0x6400 | c = 1024 + c, exact), a paired subtract of 1024 + z gives
//               c - z exactly, and a paired multiply by s rounds s (c - z) once to
//               binary16, the value grinqh_dequant writes. After the last stage the
//               same warps read the accumulators (TMEM -> registers -> Y), two warps
//               per TMEM lane quarter, each half of the token columns.
// Every wait on an mbarrier is bounded by the global timer (about one second);
// a wait that gives up sets bit 0 of the status word and the CTA skips the rest
// of its work, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace grinqh {
namespace {

constexpr int kPM = 128;                       // output columns per CTA (MMA M)
constexpr int kPN = 256;                       // tokens per CTA (MMA N)
constexpr int kPK = 64;                        // k rows per stage (four MMAs of K = 16)
constexpr int kPStages = 4;
constexpr int kPABytes = kPM * kPK * 2;        // 16 KB of binary16 weights per stage
constexpr int kPBBytes = kPN * kPK * 2;        // 32 KB of binary16 activations per stage
constexpr int kPRebuildWarps = 8;           // 8 k rows of a stage each
constexpr int kPAhead = 3;                  // stages a rebuild lane loads ahead
constexpr int kPThreads = 32 * (2 + kPRebuildWarps);

struct PfSync {
  unsigned long long full_a[kPStages];   // one arrival per rebuild warp
  unsigned long long full_b[kPStages];   // 1 arrival + the TMA's bytes
  unsigned long long empty[kPStages];    // the MMAs that read the stage have completed
  unsigned long long accum;              // every MMA of the CTA has completed
  uint32_t tmem;                         // base address of the accumulator columns
  uint32_t failed;                       // some wait of this CTA gave up
};

// Stages and shared memory of a CTA with kHalves token halves of 256.
template <int kHalves>
struct PfGeom {
  static constexpr int kStages = kHalves == 1 ? 4 : 2;
  static constexpr int kBStage = kHalves * kPBBytes;
  static constexpr int kTokens = kHalves * kPN;
  static constexpr size_t kSmem = 1024 + (size_t)kStages * (kPABytes + kBStage) + sizeof(PfSync);
};
static_assert(PfGeom<1>::kSmem <= 227 * 1024 && PfGeom<2>::kSmem <= 227 * 1024, "prefill shared memory");

// 2-D tiled TMA load of box {64 k, 256 tokens} at (k0, t0) into shared memory.
__device__ __forceinline__ void tma_x(uint32_t dst, const CUtensorMap* map, int k0, int t0, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(map), "r"(k0), "r"(t0), "r"(bar)
      : "memory");
}

// Instruction descriptor of kind::f16: D fp32, A and B binary16, A (weights)
// MN-major, B (activations) K-major, N = 256, M = 128.
constexpr uint32_t kPIdesc = (1u << 4) | (1u << 15) | ((uint32_t)(kPN >> 3) << 17) | ((uint32_t)(kPM >> 4) << 24);

// One lane's words of one (row, tile) record: its two words of each plane pair
// and its group's scale | zero word.
struct PfWords {
  uint32_t p[8];
  uint32_t m;
};

template <int kBmax>
__device__ __forceinline__ void load_words(const uint8_t* __restrict__ planes, const uint8_t* __restrict__ meta, int w,
                                           PfWords& v) {
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
  v.m = __ldg(reinterpret_cast<const uint32_t*>(meta) + (w >> 2));
}

// The binary16 weights of the lane's 32 columns, fp16_rne(s (q - z)), as 16 words
// of two values (columns 2i, 2i+1).
template <int kBmax>
__device__ __forceinline__ void rebuild_half2(const PfWords& v, uint32_t (&h)[16]) {
  uint32_t R[8];
  assemble<kBmax>(v.p, R);   // byte i of R[j]: the code of column 4j+i in the 8-bit frame
  // {s, s} and {1024 + z, 1024 + z} as binary16 pairs (z is an integer <= 255)
  const uint32_t s2 = (v.m & 0xFFFFu) * 0x10001u;
  __half2 z2 = __halves2half2(__ushort_as_half((unsigned short)(v.m >> 16)), __ushort_as_half((unsigned short)(v.m >> 16)));
  z2 = __hadd2(z2, __halves2half2(__ushort_as_half((unsigned short)0x6400u), __ushort_as_half((unsigned short)0x6400u)));
  const __half2 sh = *reinterpret_cast<const __half2*>(&s2);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t q = R[j] >> (8 - kBmax);   // b_max-bit codes, one per byte
    const uint32_t lo = __byte_perm(q, 0x64646464u, 0x5140u);   // {1024 + c0, 1024 + c1}
    const uint32_t hi = __byte_perm(q, 0x64646464u, 0x7362u);   // {1024 + c2, 1024 + c3}
    const __half2 a = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&lo), z2), sh);
    const __half2 b = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&hi), z2), sh);
    h[2 * j] = *reinterpret_cast<const uint32_t*>(&a);
    h[2 * j + 1] = *reinterpret_cast<const uint32_t*>(&b);
  }
}

template <int kBmax, int kHalves, int kSplit>
__global__ void __launch_bounds__(kPThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap xmap, const uint8_t* __restrict__ packed, size_t meta_offset,
                      int T, int K, int N, int n_tiles, float* __restrict__ Y, uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t pf_smem[];
  const uint32_t raw = saddr(pf_smem);
  using G = PfGeom<kHalves>;
  constexpr int kSt = G::kStages;
  const uint32_t a0 = (raw + 1023u) & ~1023u;   // 1 KB-aligned operand ring (swizzle atoms)
  const uint32_t b0 = a0 + kSt * kPABytes;
  PfSync& sy = *reinterpret_cast<PfSync*>(pf_smem + (a0 - raw) + kSt * (kPABytes + G::kBStage));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kPM, t0 = blockIdx.y * G::kTokens;
  // with kSplit > 1 the CTAs of a cluster (along z) take consecutive ranges of the
  // K stages and add their accumulators through distributed shared memory
  const int n_k_all = (K + kPK - 1) / kPK;
  const int rank = (kSplit > 1) ? (int)blockIdx.z : 0;
  const int ks0 = (int)(((long long)n_k_all * rank) / kSplit);
  const int n_k = (int)(((long long)n_k_all * (rank + 1)) / kSplit) - ks0;   // this CTA's stages (>= 1)

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSt; ++i) {
      bar_init(saddr(&sy.full_a[i]), kPRebuildWarps);
      bar_init(saddr(&sy.full_b[i]), 1);
      bar_init(saddr(&sy.empty[i]), 1);
    }
    bar_init(saddr(&sy.accum), 1);
    sy.failed = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&sy.tmem)),
                 "r"(G::kTokens)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = sy.tmem;
  bool ok = true;

  if (warp == 0) {
    // ---------------- activations: one TMA per stage ----------------
    int issued = -1;
    for (int it = 0; it < n_k && ok; ++it) {
      const int st = it % kSt;
      ok = bar_wait(saddr(&sy.empty[st]), ((uint32_t)(it / kSt) & 1u) ^ 1u);
      if (ok && lane == 0) {
        bar_expect(saddr(&sy.full_b[st]), G::kBStage);
#pragma unroll
        for (int hh = 0; hh < kHalves; ++hh)   // token rows past T arrive as zeros
          tma_x(b0 + st * G::kBStage + hh * kPBBytes, &xmap, (ks0 + it) * kPK, t0 + hh * kPN, saddr(&sy.full_b[st]));
      }
      if (ok) issued = it;
      __syncwarp();
    }
    // the CTA's last copies have landed before anything here can end
    for (int it = (issued - kSt + 1 > 0 ? issued - kSt + 1 : 0); it <= issued; ++it)
      bar_wait(saddr(&sy.full_b[it % kSt]), (uint32_t)(it / kSt) & 1u);
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    for (int it = 0; it < n_k && ok; ++it) {
      const int st = it % kSt;
      const uint32_t ph = (uint32_t)(it / kSt) & 1u;
      ok = bar_wait(saddr(&sy.full_a[st]), ph) && bar_wait(saddr(&sy.full_b[st]), ph);
      tc_after();
      if (ok && lane == 0) {
#pragma unroll
        for (int kk = 0; kk < kPK / 16; ++kk) {
          // A: MN-major; 64-column atoms 1 KB apart along M, 8-row groups 2 KB apart along K
          const uint64_t ad = smem_desc(a0 + st * kPABytes + kk * 4096, 1024, 2048);
#pragma unroll
          for (int hh = 0; hh < kHalves; ++hh) {
            // B: K-major rows of 128 bytes, 8-row groups 1 KB apart; K = 16 is 32 bytes into the row
            const uint64_t bd = smem_desc(b0 + st * G::kBStage + hh * kPBBytes + kk * 32, 16, 1024);
            mma_f16(tmem + (uint32_t)(hh * kPN), ad, bd, kPIdesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(saddr(&sy.empty[st]));
      }
      __syncwarp();
    }
    if (ok && lane == 0) mma_commit(saddr(&sy.accum));
    __syncwarp();
  } else {
    // ---------------- weight rebuild ----------------
    // warp d = warp - 2 rebuilds k rows 8 d .. 8 d + 7 of a stage: lane = 4 (row)
    // + q; lane quarter q owns columns 32 q .. 32 q + 31 of the CTA's 128, record
    // word w = 4 (128-column slice of the tile) + q
    const int d = warp - 2, q = lane & 3;
    const int t_rec = n0 / kTileN, w = 4 * ((n0 % kTileN) / kPM) + q;
    const size_t rbytes = (size_t)record_bytes_for(kBmax);
    const int kl = 8 * d + (lane >> 2);   // this lane's k row within a stage
    // element (column c of the lane's 32, row kl): atom (kl / 8, q / 2) at
    // (2 (kl / 8) + q / 2) KB, row kl % 8 at 128 bytes each, 16-byte chunk
    // 4 (q % 2) + c / 8 stored at chunk index (chunk ^ (kl % 8))
    const uint32_t r8 = (uint32_t)(kl & 7);
    const uint32_t row_off = (uint32_t)((2 * (kl >> 3) + (q >> 1)) * 1024) + r8 * 128u;
    auto load_stage = [&](int it, PfWords& v) {
      const int k = (ks0 + it) * kPK + kl;
      if (k < K) {
        const size_t rec = (size_t)k * n_tiles + t_rec;
        load_words<kBmax>(packed + rec * rbytes, packed + meta_offset + rec * kMetaBytes, w, v);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v.p[j] = 0u;
        v.m = 0u;   // scale 0: the row's weights are +0
      }
    };
    // stage it's words sit in buf[it % kPAhead], loaded kPAhead stages before they
    // are needed (the loop is unrolled by kPAhead so the buffers stay in registers)
    PfWords buf[kPAhead];
#pragma unroll
    for (int u = 0; u < kPAhead; ++u)
      if (u < n_k) load_stage(u, buf[u]);
    for (int i0 = 0; i0 < n_k && ok; i0 += kPAhead) {
#pragma unroll
      for (int u = 0; u < kPAhead; ++u) {
        const int it = i0 + u;
        if (it >= n_k || !ok) break;
        const int st = it % kSt;
        ok = bar_wait(saddr(&sy.empty[st]), ((uint32_t)(it / kSt) & 1u) ^ 1u);
        if (!ok) break;
        uint32_t h[16];
        rebuild_half2<kBmax>(buf[u], h);
        if (it + kPAhead < n_k) load_stage(it + kPAhead, buf[u]);
        const uint32_t row = a0 + st * kPABytes + row_off;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t chunk = ((uint32_t)(4 * (q & 1) + cc)) ^ r8;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + chunk * 16u), "r"(h[4 * cc]),
                       "r"(h[4 * cc + 1]), "r"(h[4 * cc + 2]), "r"(h[4 * cc + 3])
                       : "memory");
        }
        // the tensor core reads the tile through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(saddr(&sy.full_a[st]));
      }
    }
    // ---------------- epilogue ----------------
    // TMEM lane i of quarter (warp % 4) holds output column n0 + 32 (warp % 4) + i;
    // TMEM column j holds token t0 + j. Without a K split the warps store Y; with
    // one they store the accumulators to shared memory as D[token][column] (the
    // operand ring is free once every MMA has completed) for the cluster sum below.
    if (ok) ok = bar_wait(saddr(&sy.accum), 0u);
    tc_after();
    if (ok) {
      const int qq = warp & 3;
      const int n = n0 + 32 * qq + lane;
      constexpr int kChunks = G::kTokens / 64;   // 32-column chunks per warp: half the token columns
      const int c0 = (d >= 4) ? kChunks : 0;      // warps 6..9 take the second half
      float* dump = reinterpret_cast<float*>(pf_smem + (a0 - raw));
#pragma unroll 1
      for (int cc = c0; cc < c0 + kChunks; ++cc) {
        if (kSplit == 1 && t0 + 32 * cc >= T) break;
        uint32_t v[32];
        const uint32_t taddr = tmem + ((uint32_t)(32 * qq) << 16) + (uint32_t)(32 * cc);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
              "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
              "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
              "=r"(v[30]), "=r"(v[31])
            : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (kSplit == 1) {
          if (n < N) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int t = t0 + 32 * cc + i;
              if (t < T) Y[(size_t)t * N + n] = __uint_as_float(v[i]);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) dump[(32 * cc + i) * kPM + 32 * qq + lane] = __uint_as_float(v[i]);
        }
      }
    }
  }
  if (kSplit > 1) {
    // every thread of every CTA of the cluster takes part (no CTA leaves early):
    // rank r adds tokens [r 256 / kSplit, (r + 1) 256 / kSplit) over the ranks'
    // dumps in rank order and stores them to Y
    cluster_sync_all();
    const uint32_t dump0 = a0;
    constexpr int kSlice = kPN / kSplit;
    for (int e = threadIdx.x; e < kSlice * kPM; e += kPThreads) {
      const int tl = rank * kSlice + e / kPM, c = e % kPM;
      const uint32_t off = dump0 + (uint32_t)(tl * kPM + c) * 4u;
      float v = 0.0f;
#pragma unroll
      for (int q = 0; q < kSplit; ++q) v += ld_dsmem_f32(off, (uint32_t)q);
      const int t = t0 + tl, n = n0 + c;
      if (t < T && n < N) Y[(size_t)t * N + n] = v;
    }
    cluster_sync_all();
  }
  if (!ok) sy.failed = 1u;
  tc_before();
  __syncthreads();
  if (threadIdx.x == 0 && sy.failed) atomicOr(status, 1u);
  if (warp == 1) {
    tc_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::kTokens) : "memory");
  }
}

}  // namespace

size_t prefill_tc_smem_bytes() { return PfGeom<1>::kSmem; }

cudaError_t launch_prefill_tc(const uint16_t* X, const void* packed, int T, int K, int N, int n_tiles, int b_max,
                              float* Y, uint32_t* status, cudaStream_t st) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    cudaDriverEntryPointQueryResult qr;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr);
    if (e != cudaSuccess) return e;
    if (fn == nullptr || qr != cudaDriverEntryPointSuccess) return cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)T};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2u};
  const cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)kPN};
  const cuuint32_t estr[2] = {1u, 1u};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t meta_offset = meta_offset_for(K, n_tiles, b_max);
  // 512-token CTAs (each weight tile rebuilt once per 512 tokens) where they take
  // less time than 256-token CTAs: a wide CTA takes about 1.6x a narrow one (its MMA
  // work doubles, its rebuild does not), so compare waves x per-CTA time on this GPU
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms < 1) sms = 1;
  const long long cols = (N + kPM - 1) / kPM;
  const long long waves_n = (cols * ((T + kPN - 1) / kPN) + sms - 1) / sms;
  const long long waves_w = (cols * ((T + 2 * kPN - 1) / (2 * kPN)) + sms - 1) / sms;
  const bool wide = T > kPN && 16 * waves_w < 10 * waves_n;
  const int tokens = wide ? PfGeom<2>::kTokens : PfGeom<1>::kTokens;
  // a K split over a cluster of 2 or 4 CTAs when the grid of 256-token CTAs is small
  const long long grid_n = cols * ((T + kPN - 1) / kPN);
  const int n_k_all = (K + kPK - 1) / kPK;
  int split = 1;
  if (!wide) {
    if (4 * grid_n <= sms && n_k_all >= 4) split = 4;
    else if (2 * grid_n <= sms && n_k_all >= 2) split = 2;
  }
  const dim3 grid((unsigned)cols, (unsigned)((T + tokens - 1) / tokens), (unsigned)split);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)split;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
#define GRINQH_PF_LAUNCH(B, H, S)                                                                            \
  e = cudaFuncSetAttribute(prefill_tc_kernel<B, H, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,          \
                           (int)PfGeom<H>::kSmem);                                                           \
  if (e != cudaSuccess) return e;                                                                            \
  cfg.dynamicSmemBytes = PfGeom<H>::kSmem;                                                                   \
  e = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<B, H, S>, map, (const uint8_t*)packed, meta_offset, T, K, N, \
                         n_tiles, Y, status);
#define GRINQH_PF_CASE(B)                \
  case B:                                \
    if (wide) {                          \
      GRINQH_PF_LAUNCH(B, 2, 1)          \
    } else if (split == 4) {             \
      GRINQH_PF_LAUNCH(B, 1, 4)          \
    } else if (split == 2) {             \
      GRINQH_PF_LAUNCH(B, 1, 2)          \
    } else {                             \
      GRINQH_PF_LAUNCH(B, 1, 1)          \
    }                                    \
    break;
  switch (b_max) {
    GRINQH_PF_CASE(2)
    GRINQH_PF_CASE(4)
    GRINQH_PF_CASE(6)
    GRINQH_PF_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef GRINQH_PF_CASE
#undef GRINQH_PF_LAUNCH
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace grinqh
