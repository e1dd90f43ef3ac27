// Tensor-core encode kernels for bf16 input rows.
#include "tq_encode3_256.cuh"

namespace tq {
namespace enc3 {

namespace {

template <int K, int MODE>
cudaError_t launch_one(const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                       cudaStream_t st) {
  const int smem = (int)smem_bytes(MODE, qp.m);
  if constexpr (MODE == MODE_PROD) {
    auto kern = encode_prod_rows_kernel<__nv_bfloat16, K>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kThreads, smem, st>>>(map, qp, a);
  } else {
    auto kern = encode_tc_kernel<__nv_bfloat16, K, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kThreads, smem, st>>>(map, qp, a);
  }
  return cudaGetLastError();
}

template <int MODE>
cudaError_t by_k(const CUtensorMap& map, const QParams& qp, const Args& a, int ctas, cudaStream_t st) {
  switch (qp.k) {
    case 1: return launch_one<1, MODE>(map, qp, a, ctas, st);
    case 2: return launch_one<2, MODE>(map, qp, a, ctas, st);
    case 3: return launch_one<3, MODE>(map, qp, a, ctas, st);
    case 4:
      if constexpr (MODE != MODE_PROD) return launch_one<4, MODE>(map, qp, a, ctas, st);
      else return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <int K, int MODE>
cudaError_t launch_one256(const CUtensorMap& map, const QParams& qp, const Args& a, int ctas, cudaStream_t st) {
  const int smem = (int)smem_bytes_256();
  auto kern = encode_tc256_kernel<__nv_bfloat16, K, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<ctas, kThreads, smem, st>>>(map, qp, a);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t by_k256(const CUtensorMap& map, const QParams& qp, const Args& a, int ctas, cudaStream_t st) {
  switch (qp.k) {
    case 1: return launch_one256<1, MODE>(map, qp, a, ctas, st);
    case 2: return launch_one256<2, MODE>(map, qp, a, ctas, st);
    case 3: return launch_one256<3, MODE>(map, qp, a, ctas, st);
    case 4: return launch_one256<4, MODE>(map, qp, a, ctas, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch256_bf16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                          cudaStream_t st) {
  switch (mode) {
    case MODE_MSE_ROW: return by_k256<MODE_MSE_ROW>(map, qp, a, ctas, st);
    case MODE_MSE_BLOCK: return by_k256<MODE_MSE_BLOCK>(map, qp, a, ctas, st);
    case MODE_MSE_ROW_U: return by_k256<MODE_MSE_ROW_U>(map, qp, a, ctas, st);
    case MODE_MSE_BLOCK_U: return by_k256<MODE_MSE_BLOCK_U>(map, qp, a, ctas, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_bf16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                      cudaStream_t st) {
  switch (mode) {
    case MODE_MSE_ROW: return by_k<MODE_MSE_ROW>(map, qp, a, ctas, st);
    case MODE_MSE_BLOCK: return by_k<MODE_MSE_BLOCK>(map, qp, a, ctas, st);
    case MODE_MSE_ROW_U: return by_k<MODE_MSE_ROW_U>(map, qp, a, ctas, st);
    case MODE_MSE_BLOCK_U: return by_k<MODE_MSE_BLOCK_U>(map, qp, a, ctas, st);
    default: return by_k<MODE_PROD>(map, qp, a, ctas, st);
  }
}

}  // namespace enc3
}  // namespace tq
