// Launchers of the thread-per-vector encode kernels, one translation unit
// per input dtype (tq_enc2_f16.cu, tq_enc2_bf16.cu, tq_enc2_f32.cu).
#pragma once

#include <cuda_runtime.h>

#include "tq_encode2.cuh"

namespace tq {
namespace enc2 {

cudaError_t launch_f16(int dp, int mode, const QParams& qp, const SignMasks& sg, const Args& a,
                       size_t smem, int ctas, cudaStream_t st);
cudaError_t launch_bf16(int dp, int mode, const QParams& qp, const SignMasks& sg, const Args& a,
                        size_t smem, int ctas, cudaStream_t st);
cudaError_t launch_f32(int dp, int mode, const QParams& qp, const SignMasks& sg, const Args& a,
                       size_t smem, int ctas, cudaStream_t st);

}  // namespace enc2
}  // namespace tq
