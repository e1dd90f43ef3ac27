// fp32 GEMM C[M][N] = A[M][K] * B[N][K]^T (row-major; A rows lda apart), used
// by the dense-rotation path: y = x Pi^T (Pi row-major, y = Pi x per vector),
// z = r S^T, and the query side q' = Pi q, u = S q'.  Each output sums its K
// products in ascending k order.  SIMT with 128x128 CTA tiles, 8x8 outputs per thread, K tiles of
// 16 staged through shared memory.  M, N, K arbitrary (bounds-checked).
#pragma once

#include "tq_device.cuh"

namespace tq {

constexpr int kGemmBM = 128, kGemmBN = 128, kGemmBK = 16;

template <bool kStridedA>
__global__ void __launch_bounds__(256) gemm_abt_f32_kernel(const float* __restrict__ A,
                                                           const float* __restrict__ B,
                                                           float* __restrict__ C, int M, int N,
                                                           int K, int lda) {
  __shared__ float As[kGemmBK][kGemmBM + 4];
  __shared__ float Bs[kGemmBK][kGemmBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 8 x 8 outputs each
  const int m0 = blockIdx.y * kGemmBM, n0 = blockIdx.x * kGemmBN;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kGemmBK) {
    // 128 rows x 16 k per operand = 2048 values, 8 per thread
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = tid + 256 * r;
      const int row = e / kGemmBK, kk = e % kGemmBK;
      const int gm = m0 + row, gn = n0 + row, gk = k0 + kk;
      As[kk][row] = (gm < M && gk < K) ? A[(size_t)gm * (kStridedA ? lda : K) + gk] : 0.f;
      Bs[kk][row] = (gn < N && gk < K) ? B[(size_t)gn * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGemmBK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty * 8 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx * 8 + j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + ty * 8 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + tx * 8 + j;
      if (gn < N) C[(size_t)gm * N + gn] = acc[i][j];
    }
  }
}

inline cudaError_t gemm_abt_f32(const float* A, const float* B, float* C, int M, int N, int K,
                                cudaStream_t st, int lda = -1) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + kGemmBN - 1) / kGemmBN, (M + kGemmBM - 1) / kGemmBM);
  if (lda < 0 || lda == K)
    gemm_abt_f32_kernel<false><<<grid, 256, 0, st>>>(A, B, C, M, N, K, K);
  else
    gemm_abt_f32_kernel<true><<<grid, 256, 0, st>>>(A, B, C, M, N, K, lda);
  return cudaGetLastError();
}

}  // namespace tq
