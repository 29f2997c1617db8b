// The dense product of the prefill path: after the weights are dequantised at
// full width (dequant_kernel), prefill is a plain fp16 GEMM with fp32
// accumulation, done by cuBLAS on the caller's stream.
//
// Paper: "GRINQH" Section 4, "Prefill vs. Decoding Evaluation": the kernel
// handles prefill by unpacking the weights at full (b_max) precision and
// performing a dense matrix-matrix product.
//
// One cuBLAS handle per device, created on first use with that device current
// (cuBLAS allocates the handle's own resources then) and kept until exit; a
// mutex serialises setting the handle's stream and enqueueing the GEMM.
#include <cublas_v2.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kernels.h"

namespace grinqh {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
cublasHandle_t g_handle[kMaxDevices] = {};
}  // namespace

cudaError_t launch_prefill_gemm(const uint16_t* X, const uint16_t* W16, float* Y, int T, int K, int N,
                                cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_handle[dev] == nullptr) {
    if (cublasCreate(&g_handle[dev]) != CUBLAS_STATUS_SUCCESS) {
      g_handle[dev] = nullptr;
      return cudaErrorUnknown;
    }
  }
  cublasHandle_t h = g_handle[dev];
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return cudaErrorUnknown;
  // Row-major Y[T][N] = X[T][K] . W[K][N] is column-major Y^T (N x T) = W^T (N x K) . X^T (K x T).
  const float alpha = 1.0f, beta = 0.0f;
  const cublasStatus_t cs = cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, N, T, K, &alpha, W16, CUDA_R_16F, N, X,
                                         CUDA_R_16F, K, &beta, Y, CUDA_R_32F, N, CUBLAS_COMPUTE_32F,
                                         CUBLAS_GEMM_DEFAULT);
  return cs == CUBLAS_STATUS_SUCCESS ? cudaSuccess : cudaErrorUnknown;
}

}  // namespace grinqh
