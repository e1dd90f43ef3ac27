// Device helpers shared by libtq's kernels (one translation unit: tq_kernels.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Residual norms: fp32, or fp16 storage behind the same pointer (QParams::rnorm_f16).
__device__ __forceinline__ void put_rnorm(float* p, int64_t i, float v, int f16) {
  if (f16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else p[i] = v;
}
__device__ __forceinline__ float get_rnorm(const float* p, int64_t i, int f16) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(p)[i]) : p[i];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Unnormalized Walsh-Hadamard transform (Sylvester / natural order) of a
// vector of 32*A values spread over a warp: lane l holds coordinates 32a + l
// in v[a].  Cross-lane stages (h = 1..16) use shuffles; stages h = 32, 64, ...
// pair registers.  All stages commute, so the order is immaterial.
template <int A>
__device__ __forceinline__ void warp_fwht(float (&v)[A], int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int a = 0; a < A; ++a) {
      const float other = __shfl_xor_sync(0xffffffffu, v[a], h);
      v[a] = upper ? (other - v[a]) : (v[a] + other);
    }
  }
#pragma unroll
  for (int s = 1; s < A; s <<= 1) {
#pragma unroll
    for (int a = 0; a < A; ++a) {
      if ((a & s) == 0) {
        const float x = v[a], y = v[a + s];
        v[a] = x + y;
        v[a + s] = x - y;
      }
    }
  }
}

// D sign flip: coordinate j negated when bit j of dmask is set.
template <int A>
__device__ __forceinline__ void apply_signs(float (&v)[A], const uint32_t* dmask, int lane) {
#pragma unroll
  for (int a = 0; a < A; ++a) {
    if ((dmask[a] >> lane) & 1u) v[a] = -v[a];
  }
}

__device__ __forceinline__ int quantize_index(float y, const float* bnd, int nb) {
  // #{k : B_k < y} -- nearest centroid with ties to the lower cell.
  int idx = 0;
#pragma unroll
  for (int k = 0; k < 15; ++k) {
    if (k < nb) idx += (bnd[k] < y) ? 1 : 0;
  }
  return idx;
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

}  // namespace tq
