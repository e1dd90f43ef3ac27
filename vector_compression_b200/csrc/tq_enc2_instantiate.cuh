// Instantiation helpers for the thread-per-vector encode kernels.
#pragma once

#include "tq_enc2_launch.h"

namespace tq {
namespace enc2 {

template <int DP, typename T, int K, int MODE>
cudaError_t launch_enc2(const QParams& qp, const SignMasks& sg, const Args& a,
                        size_t smem, int ctas, cudaStream_t st) {
  auto kern = encode_kernel<DP, T, K, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<ctas, kThreads, smem, st>>>(qp, sg, a);
  return cudaGetLastError();
}

template <int DP, typename T, int MODE>
cudaError_t enc2_by_k(const QParams& qp, const SignMasks& sg, const Args& a, size_t smem,
                      int ctas, cudaStream_t st) {
  switch (qp.k) {
    case 1: return launch_enc2<DP, T, 1, MODE>(qp, sg, a, smem, ctas, st);
    case 2: return launch_enc2<DP, T, 2, MODE>(qp, sg, a, smem, ctas, st);
    case 3: return launch_enc2<DP, T, 3, MODE>(qp, sg, a, smem, ctas, st);
    case 4:
      if (MODE != MODE_PROD) return launch_enc2<DP, T, 4, MODE>(qp, sg, a, smem, ctas, st);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <int DP, typename T>
cudaError_t enc2_by_mode(int mode, const QParams& qp, const SignMasks& sg, const Args& a,
                         size_t smem, int ctas, cudaStream_t st) {
  switch (mode) {
    case MODE_MSE_ROW: return enc2_by_k<DP, T, MODE_MSE_ROW>(qp, sg, a, smem, ctas, st);
    case MODE_MSE_BLOCK: return enc2_by_k<DP, T, MODE_MSE_BLOCK>(qp, sg, a, smem, ctas, st);
    case MODE_MSE_ROW_U: return enc2_by_k<DP, T, MODE_MSE_ROW_U>(qp, sg, a, smem, ctas, st);
    case MODE_MSE_BLOCK_U: return enc2_by_k<DP, T, MODE_MSE_BLOCK_U>(qp, sg, a, smem, ctas, st);
    default: return enc2_by_k<DP, T, MODE_PROD>(qp, sg, a, smem, ctas, st);
  }
}


template <typename T>
cudaError_t launch_dtype(int dp, int mode, const QParams& qp, const SignMasks& sg, const Args& a,
                         size_t smem, int ctas, cudaStream_t st) {
  if (dp == 128) return enc2_by_mode<128, T>(mode, qp, sg, a, smem, ctas, st);
  if (dp == 256) return enc2_by_mode<256, T>(mode, qp, sg, a, smem, ctas, st);
  return cudaErrorInvalidValue;
}

}  // namespace enc2
}  // namespace tq
