// Internal definitions shared by libtq's host code and CUDA kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/tq.h"

namespace tq {

constexpr int kMaxLevels = 16;      // 2^4 code levels
constexpr int kMaxHadamard = 256;   // largest d_pad for the Hadamard rotation
constexpr int kMaxDim = 1536;       // largest vector dimension

// Quantizer description passed to kernels by value.
struct QParams {
  int d;          // vector dimension
  int d_pad;      // rotated dimension
  int k;          // code bits per coordinate (b for MSE, b - 1 for PROD)
  int m;          // QJL rows (PROD) or 0
  int rot;        // tq_rot
  int code_words; // k * ceil(d_pad / 32): ROW words per vector
  int sign_words; // m / 32
  int unbiased;   // Q_MSE with the unbiased (EDEN) per-vector scale in place of the norm
  int rnorm_f16;  // residual norms stored as fp16 (uint16 storage behind the float* arguments)
  float inv_sqrt_dpad;
  float kappa;    // sqrt(pi/2) / m
  float centroids[kMaxLevels];
  float boundaries[kMaxLevels];             // 2^k - 1 used
  uint32_t dmask[kMaxHadamard / 32];        // bit j set <=> D_j = -1
  const float* S;      // device [m][d_pad] fp32
  const float* St;     // device [d_pad][m] fp32 (S transposed)
  const uint16_t* S16; // device [m][d_pad] fp16 bits
  const float* Pi;     // device [d][d] fp32 (DENSE), y = Pi x
  const uint16_t* Pi2; // device [d][2 d] fp16 bits (DENSE): [hi | lo] of 2^8 Pi
};

}  // namespace tq

struct tq_params {
  tq::QParams q;
  int bits;            // total budget b
  int mode;            // tq_mode
  int device;
  void* dev_S;
  void* dev_St;
  void* dev_S16;
  void* dev_Pi;
  void* dev_Pi2;
  float host_centroids[tq::kMaxLevels];
  float host_boundaries[tq::kMaxLevels];
  float* host_Pi;      // d*d, DENSE only
};

namespace tq {

// Host-side numerical routines (tq_host.cpp).
int solve_codebook(int d, int bits, double* centroids, double* boundaries);
int householder_rotation(int d, const double* G, double* Pi);

// Kernel launchers (the .cu files).  All return cudaError_t as int.
int launch_encode(const QParams& qp, bool prod, const void* x, int dt, int64_t n_vec, int64_t ld,
                  int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                  float* norms, float* rnorms, void* ws, void* stream);
int launch_decode(const QParams& qp, int layout, const uint32_t* codes, const uint32_t* signs,
                  const float* norms, const float* rnorms, int64_t n_vec, int64_t seg_len,
                  int64_t seg_cap, float* out, int64_t ldo, void* stream);
int launch_query_prep(const QParams& qp, const float* q, int64_t nq, int64_t ldq, float* qrot,
                      float* u, void* stream);
int launch_scores(const QParams& qp, const float* qrot, const float* u, int64_t nq,
                  const uint32_t* codes, const uint32_t* signs, const float* norms,
                  const float* rnorms, int64_t n_vec, float* scores, void* stream);
int launch_topk(const float* scores, int64_t nq, int64_t n_vec, int topk, float* top_s,
                int64_t* top_i, void* stream);
size_t attention_workspace(const QParams& kp, const QParams& vp, int L, int B, int Hq, int Hkv,
                           int64_t seq, int* chunk_out, int* n_chunks_out);
int launch_decode_attention(const QParams& kp, const QParams& vp, const float* q, int L, int B,
                            int Hq, int Hkv, int64_t seq, int64_t cap, float scale,
                            const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                            const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                            float* out, void* ws, void* stream);
int read_and_clear_device_error(void* stream, unsigned* err);

}  // namespace tq
