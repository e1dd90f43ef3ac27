// Split-precision fp32 products on the tcgen05 tensor cores (tq_gemm_tc.cu),
// used by the dense-rotation encoder: y = Pi x (TurboQuant blog notes, the
// random rotation of Q_MSE) and z = S r (the QJL projection of Q_prod's
// residual), both dense contractions over a row of d values.
//
// An fp32 operand v is carried as two fp16 values, hi = fp16(2^8 v) and
// lo = fp16(2^8 v - hi) (22 significant bits in all), and a product as the
// sum of fp16 products hi.hi + hi.lo + lo.hi (the lo.lo term is below
// 2^-22 of the product); S is exact in fp16 and needs only r_hi.S + r_lo.S.
// The tensor cores' fp32 accumulation drifts with the number of MMAs that add
// into one accumulator (measured here on B200: the error of y grows about
// linearly with the chain length, as a truncating add would), and the QJL
// signs amplify a relative error of y by |S y| / rho.  So every chunk of
// kKC = 64 columns of K (all terms of the chunk, the small lo terms first)
// accumulates into a fresh TMEM accumulator, and the chunk sums are added in
// fp32 with round-to-nearest on the CUDA cores.  Measured at d = m = 1536
// against fp64 (chunks done as separate products): y within 0.11 of the code
// window 1e-5 / sqrt(d) and z within 0.43 of the sign window 1e-5 rho when
// formed from that y (one 288-MMA chain: 6.6 and more; a plain fp32 GEMM:
// 1.1 and 2.1).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {
namespace gemm_tc {

constexpr int kBM = 128;  // rows per tile (MMA M)
constexpr int kBN = 128;  // columns per tile (MMA N)
constexpr int kBK = 64;   // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int kKC = 64;   // K per accumulation chunk (see below)
constexpr float kSplitScale = 256.0f;  // 2^8: keeps the lo parts of unit-scale rows normal in fp16

// C[M][N] (fp32, row stride ldc) = scale * sum over terms t of
//   A[:, a_off[t] .. a_off[t] + K) * B[:, b_off[t] .. b_off[t] + K)^T
// with A fp16 [M][lda] and B fp16 [N][ldb] row-major (K contiguous).  Within
// each K chunk the terms are added in the order given: list the small ones
// first.
struct Problem {
  const uint16_t* A;
  int64_t lda;  // elements
  int64_t M;
  const uint16_t* B;
  int64_t ldb;  // elements
  int N, K;
  int nterms;  // 1..3
  int a_off[3], b_off[3];
  float scale;
  float* C;
  int64_t ldc;  // elements
};

// Shapes the kernel covers: N a multiple of 128, K a multiple of 64, at most
// four distinct column ranges among the terms' A and B operands.
bool covers(int N, int K);

// Runs the product (persistent CTAs, at most num_sms); every wait in the
// kernel is bounded (err: the device error word).  Returns an error without
// launching when the shape is not covered or a pointer or stride is not
// 16-byte aligned.
cudaError_t run(const Problem& p, unsigned* err, int num_sms, cudaStream_t st);

// Dense encode, step 1: row norms n = ||x|| into norms (segment slots) and
// A = [hi | lo] of 2^8 x / n, fp16 [nrows][2 d].  dt: TQ_F32 / TQ_F16 / TQ_BF16.
cudaError_t prep_rows(int dt, const void* x, int64_t ld, int d, int64_t seg_len, int64_t seg_cap,
                      int64_t row0, int64_t nrows, uint16_t* a2, float* norms, cudaStream_t st);

// Dense encode, step 4: A = [hi | lo] of 2^8 r for fp32 rows r [nrows][d].
cudaError_t split_rows(const float* r, int d, int64_t nrows, uint16_t* a2, cudaStream_t st);

// Host-side split of a row-major fp32 matrix [rows][cols] into
// [hi | lo] fp16 bits [rows][2 cols] (scale 2^8, round to nearest even).
void split_host(const float* v, int rows, int cols, uint16_t* out);

}  // namespace gemm_tc
}  // namespace tq
