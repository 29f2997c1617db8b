// Internal launchers of the GRINQH kernels; called by the C ABI in api.cu after
// it has validated every argument. Not part of the public interface.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace grinqh {

// Every packed-layer kernel takes the layer's planes at packed and its
// scale/zero words at packed + meta_offset (K * n_tiles * record_bytes_for(b_max)).
cudaError_t launch_pack(const float* W, int K, int N, int n_tiles, int n_groups, int b_max, void* packed,
                        cudaStream_t st);

cudaError_t launch_unpack(const void* packed, const uint8_t* bits, int K, int N, int n_tiles, int b_max,
                          uint8_t* codes, cudaStream_t st);

// Planes of given b_max-bit codes [K][N] (bits above b_max ignored); the
// scale/zero words are written as zero.
cudaError_t launch_pack_codes(const uint8_t* codes, int K, int N, int n_tiles, int b_max, void* packed,
                              cudaStream_t st);

// Full-width w_hat = s (q - z) as binary16, [K][N] row-major.
cudaError_t launch_dequant(const void* packed, int K, int N, int n_tiles, int b_max, uint16_t* out,
                           cudaStream_t st);

// Y[T][N] (fp32) = X[T][K] (fp16) . W16[K][N] (fp16), fp32 accumulation, on the
// stream (a plain library GEMM).
// The fused prefill product on the tensor cores (prefill_tc.cu): X fp16 [T][K]
// (K % 8 == 0, 16-byte aligned), Y fp32 [T][N]; bit 0 of *status is set if a
// bounded wait of the kernel gave up.
cudaError_t launch_prefill_tc(const uint16_t* X, const void* packed, int T, int K, int N, int n_tiles, int b_max,
                              float* Y, uint32_t* status, cudaStream_t st);
size_t prefill_tc_smem_bytes();

cudaError_t launch_prefill_gemm(const uint16_t* X, const uint16_t* W16, float* Y, int T, int K, int N,
                                cudaStream_t st);

struct ClassTable {
  int n;              // number of classes (1..9)
  uint8_t width[9];   // bit width of class j
};

// The batched graded product on the tensor cores (batch_tc.cu): X fp16 [T][K]
// (K % 8 == 0, 16-byte aligned), Y fp32 [T][N]; *status bit 0: a bounded wait
// gave up, bit 1: a value outside the binary16 range of the MMA operands.
cudaError_t launch_batch_tc(const uint16_t* X, int T, const void* packed, int K, int N, int n_tiles, int b_max,
                            const float* thresholds, const ClassTable& ct, float* Y, uint32_t* status,
                            cudaStream_t st);

// Largest K of launch_select: each 1024-channel block reads all of x to count
// the channels ahead of it, K^2 / 512 bytes of L2 reads per call (8 MiB here).
constexpr int kSelectMaxK = 1 << 16;
cudaError_t launch_select(const uint16_t* x, int K, const float* thresholds, const ClassTable& ct,
                          uint8_t* bits, int32_t* idx, int32_t* offsets, cudaStream_t st);

struct VmmArgs {
  int K, N, n_tiles;
  int b_max;                 // bits per stored code (2, 4, 6 or 8); records of record_bytes_for(b_max)
  const uint8_t* packed;     // planes of every record, then the scale/zero words
  size_t meta_offset;        // byte offset of the scale/zero words in packed
  const uint16_t* x;
  const int32_t* idx;
  const int32_t* offsets;
  const float* thresholds;   // fused grading only: the n_classes - 1 thresholds
  float* y;
  uint32_t* status;     // workspace: sticky error word (bit 0: a bounded wait timed out)
  float* partial;       // workspace: per-row-split partial sums [tokens][R][n_tiles * 1024]
  ClassTable ct;
  int tokens;           // batch: token t reads x + t K and writes y + t N (1 for a single vector)
  const uint8_t* lut;   // grinqh_vmm_lut: binary16 tables, 2^(b_max+2) bytes per row, heap order
};

size_t vmm_workspace_bytes(int n_tiles, int tile_n);
// Workspace of a batch of T tokens: the status word, then T sets of partials.
size_t vmm_workspace_bytes_batch(int n_tiles, int tokens);
// fused = true: the kernel grades x itself (a.thresholds) instead of reading
// a.idx / a.offsets; K <= vmm_fused_max_k().
cudaError_t launch_vmm(const VmmArgs& a, cudaStream_t st, bool fused = false);
int vmm_fused_max_k();
// Nested table codes: a.lut holds the tables; a.idx / a.offsets as for launch_vmm.
cudaError_t launch_vmm_lut(const VmmArgs& a, cudaStream_t st);

// grinqh_vmm_noalloc's shared device scratch: its size, and its address on the
// current device.
size_t vmm_noalloc_scratch_bytes();
cudaError_t vmm_noalloc_scratch(void** ptr);

// Calibration: per-sample order statistics, then the fixed-order mean.
struct CalibArgs {
  const uint16_t* X;
  int S, K, n;          // n = number of thresholds
  int lo[8], hi[8];     // ranks of the two order statistics around q_j (K-1)
  double frac[8];       // interpolation weight
  int mode[8];          // 0: interpolate, 1: theta = 0, 2: theta = +inf
  double* per_sample;   // workspace [S][n]
  float* thresholds;
};
size_t calibrate_workspace_bytes(int S, int n);
cudaError_t launch_calibrate(const CalibArgs& a, cudaStream_t st);

}  // namespace grinqh
