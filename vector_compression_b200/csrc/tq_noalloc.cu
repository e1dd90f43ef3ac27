// tq_decode_attention_noalloc: decode attention for callers that cannot
// allocate device memory.  Its scratch is a fixed device array that is part
// of the library image; the call hands that array to tq_decode_attention as
// its workspace.  Nothing here allocates: no cudaMalloc, cudaFree or
// allocating library routine.
#include <cuda_runtime.h>

#include <mutex>

#include "tq_internal.h"

namespace {

// One array per device that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
void* g_scratch_ptr[kMaxDevices];  // device address of the array, per device
std::mutex g_scratch_mu;

// Host code only sees a stand-in for the array's name, not a device address:
// look the address up once per device, with that device current.
tq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return TQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
