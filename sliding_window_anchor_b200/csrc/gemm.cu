// gemm.cu — the plain BF16 projections (a1: x·W_qkvᵀ, a6: o·W_oᵀ), FP32
// accumulation, BF16 output (or FP32 for a1 fused with the scorer's W1·x).
// These are library GEMMs (cuBLAS) with no fused epilogue; the norm/RoPE and
// state writes that follow run in k_post_proj.
#include <cublas_v2.h>

#include <mutex>

#include "common.cuh"

namespace er {

namespace {
std::mutex g_mu;
cublasHandle_t g_handle[64] = {nullptr};

// Y[M,N] (row stride ldy) = X[M,K] · W[N,K]ᵀ, row-major, BF16 operands, FP32
// accumulate, output type ytype.
int gemm_xwt(const uint16_t* X, const uint16_t* W, void* Y, cudaDataType_t ytype, int M, int N,
             int K, int ldy, cudaStream_t st) {
  if (M <= 0) return ER_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ER_ECUDA;
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_handle[dev]) {
    if (cublasCreate(&g_handle[dev]) != CUBLAS_STATUS_SUCCESS) return ER_ECUDA;
    cublasSetMathMode(g_handle[dev], CUBLAS_DEFAULT_MATH);
  }
  cublasHandle_t h = g_handle[dev];
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return ER_ECUDA;
  const float alpha = 1.f, beta = 0.f;
  // column-major view: Yᵀ[N,M] = W[N,K] · Xᵀ[K,M]
  cublasStatus_t s = cublasGemmEx(h, CUBLAS_OP_T, CUBLAS_OP_N, N, M, K, &alpha, W, CUDA_R_16BF, K,
                                  X, CUDA_R_16BF, K, &beta, Y, ytype, ldy,
                                  CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
  return s == CUBLAS_STATUS_SUCCESS ? ER_OK : ER_ECUDA;
}
}  // namespace

// Y[M,N] = X[M,K] · W[N,K]ᵀ, row-major, BF16 in/out, FP32 accumulate.
int gemm_bf16_xwt(const uint16_t* X, const uint16_t* W, uint16_t* Y, int M, int N, int K,
                  cudaStream_t st) {
  return gemm_xwt(X, W, Y, CUDA_R_16BF, M, N, K, N, st);
}

// The same with FP32 output rows of stride ldy >= N (the fused q/k/v + W1-term
// projection: the scorer's hidden pre-activations need the FP32 sums).
int gemm_bf16_xwt_f32(const uint16_t* X, const uint16_t* W, float* Y, int M, int N, int K,
                      int ldy, cudaStream_t st) {
  return gemm_xwt(X, W, Y, CUDA_R_32F, M, N, K, ldy, st);
}

}  // namespace er
