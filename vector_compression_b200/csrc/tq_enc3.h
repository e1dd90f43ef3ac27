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

enum { MODE_MSE_ROW = 0, MODE_MSE_BLOCK = 1, MODE_PROD = 2 };

struct Args {
  int64_t n_vec, seg_len, seg_cap, n_tiles;
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
cudaError_t launch_bf16(int mode, const CUtensorMap& map, const QParams& qp, const Args& a, int ctas,
                        cudaStream_t st);

// Runs the request on the tensor-core encoder if it covers it (Hadamard
// rotation with d_pad = 128, fp16/bf16 rows 16-byte aligned, segments of a
// multiple of 32 vectors, Q_prod with m in {64, 128} and k <= 3, Q_MSE k <= 4)
// and returns true with the launch status in *err; returns false otherwise.
bool try_encode(const QParams& qp, bool prod, const void* x, int dt, int64_t n_vec, int64_t ld,
                int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                float* norms, float* rnorms, unsigned* err_word, int num_sms, cudaStream_t st,
                cudaError_t* err);

}  // namespace enc3
}  // namespace tq
