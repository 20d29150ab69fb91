// Projection GEMM on CUDA cores, C[M,N] = A[M,K] * B[N,K]^T with fp32 accumulation.
// This is the float32 path of the layer (float32 configs must match the oracle to 1e-4,
// which tf32 tensor cores cannot), and also serves bf16 shapes the tensor-core kernel does
// not take (K not a multiple of 8).
#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T *__restrict__ A,
                                                        const T *__restrict__ B,
                                                        T *__restrict__ C, int M, int N, int K) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      const int m = m0 + r, n = n0 + r, k = k0 + c;
      As[c][r] = (m < M && k < K) ? to_f32(A[static_cast<size_t>(m) * K + k]) : 0.f;
      Bs[c][r] = (n < N && k < K) ? to_f32(B[static_cast<size_t>(n) * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) C[static_cast<size_t>(m) * N + n] = from_f32<T>(acc[i][j]);
    }
  }
}

}  // namespace

cudaError_t gemm_simt(int bf16, const void *A, const void *B, void *C, int M, int N, int K,
                      cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
  if (bf16)
    gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(A), static_cast<const __nv_bfloat16 *>(B),
        static_cast<__nv_bfloat16 *>(C), M, N, K);
  else
    gemm_simt_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(A),
                                                  static_cast<const float *>(B),
                                                  static_cast<float *>(C), M, N, K);
  return cudaGetLastError();
}

}  // namespace cca
