// C ABI of the GRINQH library: argument validation on the host, then launches.
// Every check happens before anything is enqueued, so a rejected call leaves the
// stream untouched. See include/grinqh.h for the contract of each call.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/grinqh.h"
#include "common.cuh"
#include "kernels.h"

using namespace grinqh;

namespace {

constexpr int64_t kMaxDim = int64_t(1) << 24;
constexpr int64_t kMaxElems = int64_t(1) << 34;
constexpr int32_t kMaxTokens = 65535;   // tokens of a batched call: one grid dimension

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

grinqh_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GRINQH_OK : GRINQH_ERR_CUDA; }

bool valid_classes(const uint8_t* classes, int32_t n) {
  if (!classes || n < 1 || n > GRINQH_MAX_CLASSES) return false;
  for (int i = 0; i < n; ++i) {
    if (classes[i] > 8) return false;
    if (i > 0 && classes[i] <= classes[i - 1]) return false;
  }
  return true;
}

bool layout_ok(const grinqh_layout* L) {
  if (!L) return false;
  grinqh_layout ref;
  if (grinqh_layout_init_bmax(L->K, L->N, L->b_max, &ref) != GRINQH_OK) return false;
  return std::memcmp(&ref, L, sizeof(ref)) == 0;
}

// Every class width fits the layout's stored planes.
bool classes_fit(const uint8_t* classes, int32_t n, int32_t b_max) {
  for (int i = 0; i < n; ++i)
    if (classes[i] > b_max) return false;
  return true;
}

ClassTable table(const uint8_t* classes, int32_t n) {
  ClassTable t{};
  t.n = n;
  for (int i = 0; i < n; ++i) t.width[i] = classes[i];
  return t;
}

// Maximum-entropy distribution p_i ~ exp(lam * b_i) with mean target (host).
void gibbs(const uint8_t* b, int m, double lam, double* p) {
  const double c = lam >= 0.0 ? (double)b[m - 1] : (double)b[0];
  double z = 0.0;
  for (int i = 0; i < m; ++i) {
    p[i] = std::exp(lam * ((double)b[i] - c));
    z += p[i];
  }
  for (int i = 0; i < m; ++i) p[i] /= z;
}

double mean_width(const uint8_t* b, int m, const double* p) {
  double s = 0.0;
  for (int i = 0; i < m; ++i) s += p[i] * (double)b[i];
  return s;
}

}  // namespace

extern "C" {

const char* grinqh_version(void) { return "grinqh-b200 0.1.0 (sm_100a)"; }

const char* grinqh_status_string(grinqh_status s) {
  switch (s) {
    case GRINQH_OK: return "ok";
    case GRINQH_ERR_INVALID_ARG: return "invalid argument";
    case GRINQH_ERR_ALIGNMENT: return "misaligned pointer";
    case GRINQH_ERR_UNSUPPORTED: return "unsupported";
    case GRINQH_ERR_WORKSPACE: return "workspace missing or too small";
    case GRINQH_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

grinqh_status grinqh_layout_init(int32_t K, int32_t N, grinqh_layout* out) {
  return grinqh_layout_init_bmax(K, N, kPlanes, out);
}

grinqh_status grinqh_layout_init_bmax(int32_t K, int32_t N, int32_t b_max, grinqh_layout* out) {
  if (!out) return GRINQH_ERR_INVALID_ARG;
  if (b_max != 2 && b_max != 4 && b_max != 6 && b_max != 8) return GRINQH_ERR_INVALID_ARG;
  if (K < 1 || N < 1 || K > kMaxDim || N > kMaxDim) return GRINQH_ERR_INVALID_ARG;
  if ((int64_t)K * N > kMaxElems) return GRINQH_ERR_INVALID_ARG;
  grinqh_layout L;
  std::memset(&L, 0, sizeof(L));
  L.K = K;
  L.N = N;
  L.n_groups = (N + GRINQH_GROUP - 1) / GRINQH_GROUP;
  L.tile_n = kTileN;
  L.n_tiles = (N + kTileN - 1) / kTileN;
  L.record_bytes = record_bytes_for(b_max);
  L.b_max = b_max;
  L.reserved = 0;
  L.packed_bytes = (int64_t)K * L.n_tiles * (L.record_bytes + kMetaBytes);
  *out = L;
  return GRINQH_OK;
}

grinqh_status grinqh_pack(const grinqh_layout* layout, const float* W, void* packed, void* stream) {
  if (!layout_ok(layout) || !W || !packed) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(packed, 16)) return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  return cuda_status(launch_pack(W, L.K, L.N, L.n_tiles, L.n_groups, L.b_max, packed, (cudaStream_t)stream));
}

grinqh_status grinqh_unpack_codes(const grinqh_layout* layout, const void* packed, const uint8_t* bits,
                                  uint8_t* codes, void* stream) {
  if (!layout_ok(layout) || !packed || !codes) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16)) return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  return cuda_status(launch_unpack(packed, bits, L.K, L.N, L.n_tiles, L.b_max, codes, (cudaStream_t)stream));
}

grinqh_status grinqh_dequant(const grinqh_layout* layout, const void* packed, uint16_t* W16, void* stream) {
  if (!layout_ok(layout) || !packed || !W16) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(W16, 16)) return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  return cuda_status(launch_dequant(packed, L.K, L.N, L.n_tiles, L.b_max, W16, (cudaStream_t)stream));
}

grinqh_status grinqh_prefill(const grinqh_layout* layout, const void* packed, const uint16_t* X, int32_t T,
                             float* Y, uint16_t* W16, void* stream) {
  if (!layout_ok(layout) || !packed || !X || !Y || !W16) return GRINQH_ERR_INVALID_ARG;
  if (T < 1 || T > kMaxDim) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(W16, 16) || !aligned(X, 2) || !aligned(Y, 4)) return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  cudaError_t e = launch_dequant(packed, L.K, L.N, L.n_tiles, L.b_max, W16, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_prefill_gemm(X, W16, Y, T, L.K, L.N, (cudaStream_t)stream);
  return cuda_status(e);
}

grinqh_status grinqh_prefill_tc(const grinqh_layout* layout, const void* packed, const uint16_t* X, int32_t T,
                                float* Y, uint32_t* status, void* stream) {
  if (!layout_ok(layout) || !packed || !X || !Y || !status) return GRINQH_ERR_INVALID_ARG;
  if (T < 1 || T > kMaxDim) return GRINQH_ERR_INVALID_ARG;
  const grinqh_layout& L = *layout;
  if (L.K % 8 != 0) return GRINQH_ERR_UNSUPPORTED;   // the TMA row pitch of X is a multiple of 16 bytes
  if ((T + 255) / 256 > 65535) return GRINQH_ERR_UNSUPPORTED;   // token tiles on the grid's y axis
  if (!aligned(packed, 16) || !aligned(X, 16) || !aligned(Y, 4) || !aligned(status, 16)) return GRINQH_ERR_ALIGNMENT;
  return cuda_status(launch_prefill_tc(X, packed, T, L.K, L.N, L.n_tiles, L.b_max, Y, status, (cudaStream_t)stream));
}

grinqh_status grinqh_maxent_distribution(const uint8_t* classes, int32_t n_classes, double target_bits,
                                         double* P) {
  if (!valid_classes(classes, n_classes) || !P) return GRINQH_ERR_INVALID_ARG;
  const double lo = classes[0], hi = classes[n_classes - 1];
  if (!(target_bits >= lo && target_bits <= hi)) return GRINQH_ERR_INVALID_ARG;
  for (int i = 0; i < n_classes; ++i) P[i] = 0.0;
  if (target_bits == hi) { P[n_classes - 1] = 1.0; return GRINQH_OK; }
  if (target_bits == lo) { P[0] = 1.0; return GRINQH_OK; }
  double p[GRINQH_MAX_CLASSES];
  // bracket lambda: mean(L) > target > mean(-L)
  double Lb = 1.0;
  for (int it = 0; it < 64; ++it) {
    gibbs(classes, n_classes, Lb, p);
    const double up = mean_width(classes, n_classes, p);
    gibbs(classes, n_classes, -Lb, p);
    const double dn = mean_width(classes, n_classes, p);
    if (up > target_bits && dn < target_bits) break;
    Lb *= 2.0;
  }
  double a = -Lb, c = Lb;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (a + c);
    if (mid == a || mid == c) break;
    gibbs(classes, n_classes, mid, p);
    if (mean_width(classes, n_classes, p) < target_bits) a = mid; else c = mid;
  }
  gibbs(classes, n_classes, 0.5 * (a + c), P);
  return GRINQH_OK;
}

grinqh_status grinqh_calibrate_workspace_bytes(int32_t S, int32_t n_classes, size_t* bytes) {
  if (!bytes || S < 1 || S > 65535 || n_classes < 1 || n_classes > GRINQH_MAX_CLASSES)
    return GRINQH_ERR_INVALID_ARG;
  *bytes = calibrate_workspace_bytes(S, n_classes - 1);
  return GRINQH_OK;
}

grinqh_status grinqh_calibrate(const uint16_t* X, int32_t S, int32_t K, const uint8_t* classes,
                               int32_t n_classes, const double* P, double target_bits, float* thresholds,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (S < 1 || S > 65535 || K < 1 || K > kMaxDim) return GRINQH_ERR_INVALID_ARG;
  const int n = n_classes - 1;
  if (n > 0 && (!X || !thresholds)) return GRINQH_ERR_INVALID_ARG;
  double Pv[GRINQH_MAX_CLASSES];
  if (P) {
    double tot = 0.0;
    for (int i = 0; i < n_classes; ++i) {
      if (!(P[i] >= 0.0)) return GRINQH_ERR_INVALID_ARG;
      Pv[i] = P[i];
      tot += P[i];
    }
    if (std::fabs(tot - 1.0) > 1e-9) return GRINQH_ERR_INVALID_ARG;
  } else {
    const grinqh_status st = grinqh_maxent_distribution(classes, n_classes, target_bits, Pv);
    if (st != GRINQH_OK) return st;
  }
  if (n == 0) return GRINQH_OK;
  if (!aligned(X, 2) || !aligned(thresholds, 4) || !aligned(workspace, 16)) return GRINQH_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < calibrate_workspace_bytes(S, n)) return GRINQH_ERR_WORKSPACE;

  CalibArgs a{};
  a.X = X;
  a.S = S;
  a.K = K;
  a.n = n;
  a.per_sample = (double*)workspace;
  a.thresholds = thresholds;
  double q = 0.0;
  for (int j = 1; j <= n; ++j) {
    q += Pv[j - 1];   // q_j = p_0 + ... + p_{j-1}, summed in ascending order
    bool tail_empty = true;
    for (int i = j; i < n_classes; ++i)
      if (Pv[i] != 0.0) tail_empty = false;
    const int jj = j - 1;
    if (tail_empty) { a.mode[jj] = 2; continue; }
    if (q == 0.0) { a.mode[jj] = 1; continue; }
    a.mode[jj] = 0;
    const double pos = q * (double)(K - 1);
    if (pos >= (double)(K - 1)) {
      a.lo[jj] = a.hi[jj] = K - 1;
      a.frac[jj] = 0.0;
    } else {
      const double fl = std::floor(pos);
      a.lo[jj] = (int)fl;
      a.hi[jj] = (a.lo[jj] + 1 < K) ? a.lo[jj] + 1 : K - 1;
      a.frac[jj] = pos - fl;
    }
  }
  return cuda_status(launch_calibrate(a, (cudaStream_t)stream));
}

grinqh_status grinqh_select(const uint16_t* x, int32_t K, const float* thresholds, const uint8_t* classes,
                            int32_t n_classes, uint8_t* bits, int32_t* idx, int32_t* offsets, void* stream) {
  if (!valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (K < 1 || K > kMaxDim) return GRINQH_ERR_INVALID_ARG;
  if (K > kSelectMaxK) return GRINQH_ERR_UNSUPPORTED;
  if (!x || !bits || !idx || !offsets || (n_classes > 1 && !thresholds)) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(idx, 4) || !aligned(offsets, 4) || (thresholds && !aligned(thresholds, 4)))
    return GRINQH_ERR_ALIGNMENT;
  return cuda_status(launch_select(x, K, thresholds, table(classes, n_classes), bits, idx, offsets,
                                   (cudaStream_t)stream));
}

grinqh_status grinqh_vmm_workspace_bytes(const grinqh_layout* layout, size_t* bytes) {
  if (!layout_ok(layout) || !bytes) return GRINQH_ERR_INVALID_ARG;
  *bytes = vmm_workspace_bytes(layout->n_tiles, layout->tile_n);
  return GRINQH_OK;
}

grinqh_status grinqh_vmm(const grinqh_layout* layout, const void* packed, const uint16_t* x, const int32_t* idx,
                         const int32_t* offsets, const uint8_t* classes, int32_t n_classes, float* y,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!layout_ok(layout) || !valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (!classes_fit(classes, n_classes, layout->b_max)) return GRINQH_ERR_INVALID_ARG;
  if (!packed || !x || !idx || !offsets || !y) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(x, 2) || !aligned(idx, 4) || !aligned(offsets, 4) || !aligned(y, 4))
    return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  const size_t need = vmm_workspace_bytes(L.n_tiles, L.tile_n);
  if (!workspace || workspace_bytes < need) return GRINQH_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return GRINQH_ERR_ALIGNMENT;
  VmmArgs a{};
  a.K = L.K;
  a.N = L.N;
  a.n_tiles = L.n_tiles;
  a.b_max = L.b_max;
  a.packed = (const uint8_t*)packed;
  a.meta_offset = meta_offset_for(L.K, L.n_tiles, L.b_max);
  a.x = x;
  a.idx = idx;
  a.offsets = offsets;
  a.y = y;
  a.status = (uint32_t*)workspace;
  a.partial = (float*)((char*)workspace + 16);
  a.ct = table(classes, n_classes);
  return cuda_status(launch_vmm(a, (cudaStream_t)stream));
}

grinqh_status grinqh_vmm_noalloc(const grinqh_layout* layout, const void* packed, const uint16_t* x,
                                 const int32_t* idx, const int32_t* offsets, const uint8_t* classes,
                                 int32_t n_classes, float* y, void* stream) {
  if (!layout_ok(layout) || !valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (!classes_fit(classes, n_classes, layout->b_max)) return GRINQH_ERR_INVALID_ARG;
  if (!packed || !x || !idx || !offsets || !y) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(x, 2) || !aligned(idx, 4) || !aligned(offsets, 4) || !aligned(y, 4))
    return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  if (vmm_workspace_bytes(L.n_tiles, L.tile_n) > vmm_noalloc_scratch_bytes()) return GRINQH_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (vmm_noalloc_scratch(&scratch) != cudaSuccess) return GRINQH_ERR_CUDA;
  VmmArgs a{};
  a.K = L.K;
  a.N = L.N;
  a.n_tiles = L.n_tiles;
  a.b_max = L.b_max;
  a.packed = (const uint8_t*)packed;
  a.meta_offset = meta_offset_for(L.K, L.n_tiles, L.b_max);
  a.x = x;
  a.idx = idx;
  a.offsets = offsets;
  a.y = y;
  a.status = (uint32_t*)scratch;
  a.partial = (float*)((char*)scratch + 16);
  a.ct = table(classes, n_classes);
  return cuda_status(launch_vmm(a, (cudaStream_t)stream));
}

grinqh_status grinqh_select_vmm(const grinqh_layout* layout, const void* packed, const uint16_t* x,
                                const float* thresholds, const uint8_t* classes, int32_t n_classes, float* y,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!layout_ok(layout) || !valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (!classes_fit(classes, n_classes, layout->b_max)) return GRINQH_ERR_INVALID_ARG;
  if (!packed || !x || !y || (n_classes > 1 && !thresholds)) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(x, 2) || !aligned(y, 4) || (thresholds && !aligned(thresholds, 4)))
    return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  if (L.K > vmm_fused_max_k()) return GRINQH_ERR_UNSUPPORTED;
  const size_t need = vmm_workspace_bytes(L.n_tiles, L.tile_n);
  if (!workspace || workspace_bytes < need) return GRINQH_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return GRINQH_ERR_ALIGNMENT;
  VmmArgs a{};
  a.K = L.K;
  a.N = L.N;
  a.n_tiles = L.n_tiles;
  a.b_max = L.b_max;
  a.packed = (const uint8_t*)packed;
  a.meta_offset = meta_offset_for(L.K, L.n_tiles, L.b_max);
  a.x = x;
  a.thresholds = thresholds;
  a.y = y;
  a.status = (uint32_t*)workspace;
  a.partial = (float*)((char*)workspace + 16);
  a.ct = table(classes, n_classes);
  return cuda_status(launch_vmm(a, (cudaStream_t)stream, true));
}

grinqh_status grinqh_vmm_batch_workspace_bytes(const grinqh_layout* layout, int32_t tokens, size_t* bytes) {
  if (!layout_ok(layout) || !bytes || tokens < 1 || tokens > kMaxTokens) return GRINQH_ERR_INVALID_ARG;
  *bytes = vmm_workspace_bytes_batch(layout->n_tiles, tokens);
  return GRINQH_OK;
}

grinqh_status grinqh_select_vmm_batch(const grinqh_layout* layout, const void* packed, const uint16_t* X,
                                      int32_t tokens, const float* thresholds, const uint8_t* classes,
                                      int32_t n_classes, float* Y, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  if (!layout_ok(layout) || !valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (!classes_fit(classes, n_classes, layout->b_max)) return GRINQH_ERR_INVALID_ARG;
  if (tokens < 1 || tokens > kMaxTokens) return GRINQH_ERR_INVALID_ARG;
  if (!packed || !X || !Y || (n_classes > 1 && !thresholds)) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(X, 2) || !aligned(Y, 4) || (thresholds && !aligned(thresholds, 4)))
    return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  if (L.K > vmm_fused_max_k()) return GRINQH_ERR_UNSUPPORTED;
  const size_t need = vmm_workspace_bytes_batch(L.n_tiles, tokens);
  if (!workspace || workspace_bytes < need) return GRINQH_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return GRINQH_ERR_ALIGNMENT;
  VmmArgs a{};
  a.K = L.K;
  a.N = L.N;
  a.n_tiles = L.n_tiles;
  a.b_max = L.b_max;
  a.packed = (const uint8_t*)packed;
  a.meta_offset = meta_offset_for(L.K, L.n_tiles, L.b_max);
  a.x = X;
  a.thresholds = thresholds;
  a.y = Y;
  a.ct = table(classes, n_classes);
  a.status = (uint32_t*)workspace;
  a.partial = (float*)((char*)workspace + 16);
  a.tokens = tokens;
  return cuda_status(launch_vmm(a, (cudaStream_t)stream, true));
}

grinqh_status grinqh_select_vmm_batch_tc(const grinqh_layout* layout, const void* packed, const uint16_t* X,
                                         int32_t tokens, const float* thresholds, const uint8_t* classes,
                                         int32_t n_classes, float* Y, uint32_t* status, void* stream) {
  if (!layout_ok(layout) || !valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (!classes_fit(classes, n_classes, layout->b_max)) return GRINQH_ERR_INVALID_ARG;
  if (tokens < 1 || tokens > kMaxTokens) return GRINQH_ERR_INVALID_ARG;
  if (!packed || !X || !Y || !status || (n_classes > 1 && !thresholds)) return GRINQH_ERR_INVALID_ARG;
  const grinqh_layout& L = *layout;
  if (L.K % 8 != 0) return GRINQH_ERR_UNSUPPORTED;   // 16-byte loads of X rows
  if (!aligned(packed, 16) || !aligned(X, 16) || !aligned(Y, 4) || !aligned(status, 16) ||
      (thresholds && !aligned(thresholds, 4)))
    return GRINQH_ERR_ALIGNMENT;
  return cuda_status(launch_batch_tc(X, tokens, packed, L.K, L.N, L.n_tiles, L.b_max, thresholds,
                                     table(classes, n_classes), Y, status, (cudaStream_t)stream));
}

grinqh_status grinqh_pack_codes(const grinqh_layout* layout, const uint8_t* codes, void* packed, void* stream) {
  if (!layout_ok(layout) || !codes || !packed) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16)) return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  return cuda_status(launch_pack_codes(codes, L.K, L.N, L.n_tiles, L.b_max, packed, (cudaStream_t)stream));
}

grinqh_status grinqh_lut_bytes(const grinqh_layout* layout, size_t* bytes) {
  if (!layout_ok(layout) || !bytes) return GRINQH_ERR_INVALID_ARG;
  *bytes = (size_t)layout->K << (layout->b_max + 2);
  return GRINQH_OK;
}

grinqh_status grinqh_vmm_lut(const grinqh_layout* layout, const void* packed, const uint16_t* lut,
                             const uint16_t* x, const int32_t* idx, const int32_t* offsets, const uint8_t* classes,
                             int32_t n_classes, float* y, void* workspace, size_t workspace_bytes, void* stream) {
  if (!layout_ok(layout) || !valid_classes(classes, n_classes)) return GRINQH_ERR_INVALID_ARG;
  if (!classes_fit(classes, n_classes, layout->b_max)) return GRINQH_ERR_INVALID_ARG;
  if (!packed || !lut || !x || !idx || !offsets || !y) return GRINQH_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(lut, 16) || !aligned(x, 2) || !aligned(idx, 4) || !aligned(offsets, 4) ||
      !aligned(y, 4))
    return GRINQH_ERR_ALIGNMENT;
  const grinqh_layout& L = *layout;
  const size_t need = vmm_workspace_bytes(L.n_tiles, L.tile_n);
  if (!workspace || workspace_bytes < need) return GRINQH_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return GRINQH_ERR_ALIGNMENT;
  VmmArgs a{};
  a.K = L.K;
  a.N = L.N;
  a.n_tiles = L.n_tiles;
  a.b_max = L.b_max;
  a.packed = (const uint8_t*)packed;
  a.meta_offset = meta_offset_for(L.K, L.n_tiles, L.b_max);
  a.lut = (const uint8_t*)lut;
  a.x = x;
  a.idx = idx;
  a.offsets = offsets;
  a.y = y;
  a.status = (uint32_t*)workspace;
  a.partial = (float*)((char*)workspace + 16);
  a.ct = table(classes, n_classes);
  return cuda_status(launch_vmm_lut(a, (cudaStream_t)stream));
}

}  // extern "C"
