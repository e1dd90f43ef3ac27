// Launch parameters shared by the tensor-core decode-attention kernels
// (tq_attn3.cu, tq_attn4.cu) and the odd-subset coefficients of a symmetric
// codebook that both use.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace tq {
namespace attn {

struct Params {
  int G;          // query heads per KV head (1..8)
  int chunk;      // tokens per chunk (multiple of 64)
  int n_chunks;
  int64_t seq, cap;
  float scale, kappa;
  const float* qrot;  // [groups * G][d_pad]
  const float* u;     // [groups * G][m]
  const uint32_t* kcodes;
  const uint32_t* ksigns;
  const float* knorms;
  const float* krnorms;  // fp32, or fp16 storage when kr16
  int kr16;
  const uint32_t* vcodes;
  const float* vnorms;
  float* part;
  unsigned* err;    // device error word (bounded waits)
  float kalpha[8];  // odd-subset coefficients of the key codebook
  float kalpha_sum;
  float valpha[8];  // and of the value codebook
  float valpha_sum;
};

// Coefficients alpha_S of C[idx] = sum_S alpha_S prod_{p in S} (2 b_p - 1)
// over the odd subsets S of the k index bits, in the order {0}, ..., {k-1},
// then the triples ({0,1,2}; for k = 4 also {0,1,3}, {0,2,3}, {1,2,3}).
void odd_feature_coefs(const float* centroids, int k, float* alpha, float* alpha_sum);

}  // namespace attn
}  // namespace tq
