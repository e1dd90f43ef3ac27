// Host-visible part of the tensor-core encoder (tq_encode3.cuh): argument
// block, tile constants and launchers (one translation unit per input dtype:
// tq_enc3_f16.cu, tq_enc3_bf16.cu; request checks in tq_enc3_host.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {
namespace enc3 {

constexpr int kDP = 128;                           // rotated dimension handled
constexpr int kRows = 128;                         // vectors per tile (MMA M)
constexpr int kStages = 4;                         // input ring depth
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;      // 320
constexpr uint32_t kTileBytes = kRows * kDP * 2;   // 32 KB of 16-bit input
constexpr uint32_t kRotBytes = kDP * kDP * 2;      // 32 KB rotation operand

// *_U: Q_MSE with the unbiased (EDEN) scale n / <y, C[idx]> stored as the norm
enum { MODE_MSE_ROW = 0, MODE_MSE_BLOCK = 1, MODE_PROD = 2, MODE_MSE_ROW_U = 3, MODE_MSE_BLOCK_U = 4 };

// Division by a fixed d (1 <= d < 2^31) of n < 2^31 as a multiply and shift:
// with s = ceil(log2 d) and M = floor(2^(32+s) / d) + 1 = 2^32 + mul, the
// product n M / 2^(32+s) exceeds n / d by less than n / 2^(32+s) < 1 / (2d),
// too little to reach the next integer, so
// floor(n / d) = (umulhi(n, mul) + n) >> s  (the sum stays below 2^32).
struct FastDiv {
  uint32_t d, mul, shift;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.shift = 0;
  while (((uint64_t)1 << f.shift) < d) ++f.shift;
  f.mul = (uint32_t)((((uint64_t)1 << (32 + f.shift)) / d) - ((uint64_t)1 << 32) + 1);
  return f;
}
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fastdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.mul) + n) >> f.shift;
}
#endif

struct Args {
  int64_t n_vec, seg_len, seg_cap, n_tiles;
  FastDiv seg_div;  // division by seg_len
  uint32_t* codes;
  uint32_t* signs;
  float* norms;
  float* rnorms;
  unsigned* err;  // device error word (bounded-wait expiry)
};

// Dynamic shared memory: [rotation H D (no swizzle, 32 KB) | S (Q_prod, m x 128
// fp16) | kStages input tiles of 32 KB] plus slack for 1024-byte alignment.
inline uint32_t smem_bytes(int mode, int m) {
  return kRotBytes + (mode == MODE_PROD ? (uint32_t)m * kDP * 2 : 0u) + kStages * kTileBytes + 1024;
}

cudaError_t launch_f16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                       cudaStream_t st);
// Q_MSE modes at d_pad = 256 (tq_encode3_256.cuh)
cudaError_t launch256_f16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                          cudaStream_t st);
cudaError_t launch256_bf16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                           cudaStream_t st);
cudaError_t launch_bf16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                        cudaStream_t st);

// Runs the request on the tensor-core encoder if it covers it (Hadamard
// rotation with d_pad = 128, or Q_MSE with d_pad = 256; fp16/bf16 rows 16-byte
// aligned, segments of a multiple of 32 vectors, Q_prod with m in {64, 128}
// and k <= 3, Q_MSE k <= 4) and returns true with the launch status in *err;
// returns false otherwise.
bool try_encode(const QParams& qp, bool prod, const void* x, int dt, int64_t n_vec, int64_t ld,
                int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                float* norms, float* rnorms, unsigned* err_word, int num_sms, cudaStream_t st,
                cudaError_t* err);

}  // namespace enc3
}  // namespace tq
