// Thread-per-vector encode kernels for __half inputs.
#include "tq_enc2_instantiate.cuh"

namespace tq {
namespace enc2 {

cudaError_t launch_f16(int dp, int mode, const QParams& qp, const SignMasks& sg, const Args& a,
                       size_t smem, int ctas, cudaStream_t st) {
  return launch_dtype<__half>(dp, mode, qp, sg, a, smem, ctas, st);
}

}  // namespace enc2
}  // namespace tq
