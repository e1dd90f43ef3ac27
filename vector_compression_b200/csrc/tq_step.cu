// tq_decode_step: one serving decode step -- append the new token's key and
// value to every (layer, batch, kv-head) cache and attend over the grown
// caches ("turboquant-pytorch" skill page, KV Cache Wrapper
// (TurboQuantKVCache): append_key / append_value as tokens are generated,
// then attention over all cached keys and MSE-reconstructed values).
//
// The new keys are Q_prod-encoded straight into slot `pos` of the ROW key
// cache (the encoder writes slot g * cap of segment g; the output pointers
// are advanced by pos slots).  The new values are Q_MSE-encoded into a small
// ROW buffer in the workspace, and a scatter kernel moves each code bit into
// bit pos % 32 of its BLOCK32 word (one thread per word, so the other 31
// tokens of the block are preserved).  Then the decode attention runs over
// pos + 1 tokens.  All launches are on `stream`, in order.
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kStepMaxG = 16;  // query heads per KV head, as tq_decode_attention
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// tmp: ROW Q_MSE codes [n][k * d_pad / 32] of the new values; thread
// (g, p, j) copies bit (j mod 32) of word (p, j / 32) into bit pos % 32 of
// the BLOCK32 word (p, j) of block pos / 32 of group g.
__global__ void scatter_block32_kernel(const uint32_t* tmp, const float* tmp_norms, int n, int k, int d_pad,
                                       int64_t pos, int64_t cap, uint32_t* vcodes, float* vnorms) {
  const int64_t total = (int64_t)n * k * d_pad;
  const int words = k * d_pad / 32;
  const uint32_t bit = 1u << (pos & 31);
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = e / (k * d_pad);
    const int pj = (int)(e - g * k * d_pad);  // p * d_pad + j
    const int p = pj / d_pad, j = pj - p * d_pad;
    const uint32_t src = tmp[g * words + p * (d_pad / 32) + j / 32];
    uint32_t* w = vcodes + (g * (cap / 32) + pos / 32) * (int64_t)(k * d_pad) + pj;
    *w = ((src >> (j & 31)) & 1u) ? (*w | bit) : (*w & ~bit);
    if (pj == 0) vnorms[g * cap + pos] = tmp_norms[g];
  }
}

}  // namespace
}  // namespace tq

namespace {

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// workspace: [attention workspace | ROW value codes of the new tokens | their norms]
size_t step_bytes(const tq_params* kp, const tq_params* vp, int L, int B, int Hq, int Hkv, int64_t pos,
                  size_t* att) {
  const int64_t n = (int64_t)L * B * Hkv;
  *att = round256(tq::attention_workspace(kp->q, vp->q, L, B, Hq, Hkv, pos + 1, nullptr, nullptr));
  return *att + round256((size_t)n * vp->q.code_words * 4) + round256((size_t)n * 4);
}

}  // namespace

extern "C" tq_status tq_decode_step_workspace_size(const tq_params* kp, const tq_params* vp, int L, int B,
                                                   int Hq, int Hkv, int64_t pos, size_t* bytes) {
  if (!kp || !vp || !bytes || L < 1 || B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || pos < 0)
    return TQ_ERR_INVALID_ARG;
  size_t att = 0;
  *bytes = step_bytes(kp, vp, L, B, Hq, Hkv, pos, &att);
  return TQ_OK;
}

extern "C" tq_status tq_decode_step(const tq_params* kp, const tq_params* vp, const float* q,
                                    const void* k_new, const void* v_new, tq_dtype dt, int L, int B,
                                    int Hq, int Hkv, int64_t pos, int64_t cap, float scale,
                                    uint32_t* kcodes, uint32_t* ksigns, float* knorms, float* krnorms,
                                    uint32_t* vcodes, float* vnorms, float* out, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (!kp || !vp || kp->mode != TQ_MODE_PROD || (vp->mode != TQ_MODE_MSE && vp->mode != TQ_MODE_MSE_UNBIASED))
    return TQ_ERR_INVALID_ARG;
  if (kp->q.d != vp->q.d || kp->q.rot != vp->q.rot) return TQ_ERR_INVALID_ARG;
  if (kp->q.rot != TQ_ROT_HADAMARD) return TQ_ERR_UNSUPPORTED;
  if (dt != TQ_F32 && dt != TQ_F16 && dt != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (L < 1 || B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0) return TQ_ERR_INVALID_ARG;
  if (Hq / Hkv > tq::kStepMaxG) return TQ_ERR_UNSUPPORTED;
  if (pos < 0 || cap % 32 != 0 || pos >= cap) return TQ_ERR_INVALID_ARG;
  if (!q || !k_new || !v_new || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms || !out)
    return TQ_ERR_INVALID_ARG;
  if (!tq::al16(q) || !tq::al16(kcodes) || !tq::al16(ksigns) || !tq::al16(vcodes) ||
      !tq::al16(out) || !tq::al16(k_new) || !tq::al16(v_new))
    return TQ_ERR_INVALID_ARG;
  size_t att = 0;
  const size_t need = step_bytes(kp, vp, L, B, Hq, Hkv, pos, &att);
  if (!ws || ws_bytes < need || !tq::al256(ws)) return TQ_ERR_WORKSPACE;
  const int64_t n = (int64_t)L * B * Hkv;
  const int d = kp->q.d;
  char* w = (char*)ws;
  uint32_t* tmp = reinterpret_cast<uint32_t*>(w + att);
  float* tmp_norms = reinterpret_cast<float*>(w + att + round256((size_t)n * vp->q.code_words * 4));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // keys: segment g of one vector -> slot g * cap, shifted by pos slots
  int e = tq::launch_encode(kp->q, true, k_new, dt, n, d, 1, cap, TQ_LAYOUT_ROW,
                            kcodes + pos * kp->q.code_words, ksigns + pos * kp->q.sign_words, knorms + pos,
                            // fp16 residual norms are 2-byte slots
                            reinterpret_cast<float*>(reinterpret_cast<char*>(krnorms) + pos * (kp->q.rnorm_f16 ? 2 : 4)),
                            nullptr, stream);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  // values: ROW codes into the workspace, then into bit pos % 32 of their blocks
  e = tq::launch_encode(vp->q, false, v_new, dt, n, d, 1, 1, TQ_LAYOUT_ROW, tmp, nullptr, tmp_norms, nullptr,
                        nullptr, stream);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  const int64_t total = n * vp->q.k * vp->q.d_pad;
  const unsigned blocks = (unsigned)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  tq::scatter_block32_kernel<<<blocks, 256, 0, st>>>(tmp, tmp_norms, (int)n, vp->q.k, vp->q.d_pad, pos, cap,
                                                     vcodes, vnorms);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  e = tq::launch_decode_attention(kp->q, vp->q, q, L, B, Hq, Hkv, pos + 1, cap, scale, kcodes, ksigns, knorms,
                                  krnorms, vcodes, vnorms, out, ws, stream);
  return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
