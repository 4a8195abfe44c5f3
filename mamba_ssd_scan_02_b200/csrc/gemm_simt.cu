// gemm_simt.cu -- reference-quality CUDA-core GEMM C[M,N] = A[M,K] . B[N,K]^T (bf16 in,
// fp32 accumulate, bf16 out).  Used for projection shapes the tensor-core GEMM does not tile.
#include "common.cuh"
#include "plan.h"

namespace ssd {
namespace {

constexpr int BM = 64, BN = 64, BK = 32;

__global__ void __launch_bounds__(256) gemm_simt_kernel(const __nv_bfloat16 *__restrict__ A, long long lda,
                                                        const __nv_bfloat16 *__restrict__ Bm, long long ldb,
                                                        __nv_bfloat16 *__restrict__ C, long long ldc,
                                                        int M, int N, int K,
                                                        const float *__restrict__ row_scale) {
  __shared__ float As[BK][BM + 1];
  __shared__ float Bs[BK][BN + 1];
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;
  const long long m0 = (long long)blockIdx.y * BM, n0 = (long long)blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, k = i % BK;
      As[k][r] = (m0 + r < M && k0 + k < K) ? __bfloat162float(A[(m0 + r) * lda + k0 + k]) : 0.f;
      Bs[k][r] = (n0 + r < N && k0 + k < K) ? __bfloat162float(Bm[(n0 + r) * ldb + k0 + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < BK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tc + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long m = m0 + tr * 4 + i, n = n0 + tc + 16 * j;
      if (m < M && n < N) C[m * ldc + n] = __float2bfloat16_rn(row_scale ? acc[i][j] * row_scale[m] : acc[i][j]);
    }
}

}  // namespace

cudaError_t launch_gemm_simt_bf16_tn(const void *A, long long lda, const void *Bm, long long ldb, void *C,
                                     long long ldc, int M, int N, int K, cudaStream_t s,
                                     const float *row_scale) {
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  gemm_simt_kernel<<<grid, 256, 0, s>>>((const __nv_bfloat16 *)A, lda, (const __nv_bfloat16 *)Bm, ldb,
                                        (__nv_bfloat16 *)C, ldc, M, N, K, row_scale);
  return cudaGetLastError();
}

}  // namespace ssd
