// tq_decode_attention_noalloc: decode attention for callers that cannot
// allocate device memory.  Its scratch is a fixed device array that is part
// of the library image; the call hands that array to tq_decode_attention as
// its workspace.  Nothing here allocates: no cudaMalloc, cudaFree or
// allocating library routine.
#include <cuda_runtime.h>

#include "tq_internal.h"

namespace {

// One array per device that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

// Host code only sees a stand-in for the array's name, not a device address.
// The address is looked up on every call, with the caller's device and
// context current, so it is always the array of the context the kernels
// will run in: a cached address would go stale after cudaDeviceReset or
// belong to another context when the caller switches contexts.  The lookup
// allocates nothing; the first lookup in a context may load the library's
// module into it, so that first call should come before any stream capture.
tq_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return TQ_ERR_CUDA;
  *out = p;
  return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_decode_attention_noalloc(
    const tq_params* kp, const tq_params* vp, const float* q, int L, int B, int Hq, int Hkv,
    int64_t seq, int64_t cap, float scale, const uint32_t* kcodes, const uint32_t* ksigns,
    const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms,
    float* out, void* stream) {
  size_t need = 0;
  tq_status s = tq_decode_attention_workspace_size(kp, vp, L, B, Hq, Hkv, seq, &need);
  if (s != TQ_OK) return s;
  if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = scratch_address(&scratch);
  if (s != TQ_OK) return s;
  return tq_decode_attention(kp, vp, q, L, B, Hq, Hkv, seq, cap, scale, kcodes, ksigns, knorms,
                             krnorms, vcodes, vnorms, out, scratch, TQ_NOALLOC_SCRATCH_BYTES,
                             stream);
}
