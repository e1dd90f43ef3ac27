// Encode kernels: TurboQuant-MSE and TurboQuant-prod.
//
// Per vector (TurboQuant blog notes, Q_MSE and the definition of Q_prod;
// explainer §6 and §8):
//   n = ||x||, y = Pi (x / n), idx_j = #{k : B_k < y_j}, codes = pack(idx);
//   Q_prod additionally: r = y - C[idx], rho = ||r||, sign bits of S r.
//
// Hadamard rotation (explainer §0.9, DRIVE's randomized Hadamard; FastVQ's
// sign-flipped Hadamard with padding): one warp per vector, lane l holding
// coordinates 32a + l; the transform runs in registers and shuffles.
// Dense rotation: the rotation and the QJL projection run as GEMMs over a
// chunk of vectors (tq_gemm.cuh), with the per-vector steps here.
#pragma once

#include "tq_device.cuh"

namespace tq {

// Shared per-CTA copy of the codebook (dynamic indexing by lane).
struct SmemCodebook {
  float c[kMaxLevels];
  float b[kMaxLevels];
};

__device__ __forceinline__ void load_codebook(SmemCodebook& cb, const QParams& qp) {
  if (threadIdx.x < kMaxLevels) {
    cb.c[threadIdx.x] = qp.centroids[threadIdx.x];
    cb.b[threadIdx.x] = qp.boundaries[threadIdx.x];
  }
}

// Quantize the rotated unit vector held by the warp (lane l: coordinates
// 32a + l in y[a]) and emit ROW code words (lane w < k*A ends with word w in
// *row_word) or accumulate BLOCK32 bits for vector slot t.  Returns idx in
// idx[a].  Coordinates >= d_pad are not present (d_pad = 32 A).
template <int A>
__device__ __forceinline__ void quantize_pack(const float (&y)[A], int (&idx)[A],
                                              const SmemCodebook& cb, int k, int lane,
                                              uint32_t* row_word, uint32_t (*blk)[A], int t,
                                              bool block_layout) {
  const int nb = (1 << k) - 1;
#pragma unroll
  for (int a = 0; a < A; ++a) idx[a] = quantize_index(y[a], cb.b, nb);
  if (block_layout) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      if (p < k) {
#pragma unroll
        for (int a = 0; a < A; ++a) blk[p][a] |= (uint32_t)((idx[a] >> p) & 1) << t;
      }
    }
  } else {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      if (p < k) {
#pragma unroll
        for (int a = 0; a < A; ++a) {
          const uint32_t w = __ballot_sync(0xffffffffu, (idx[a] >> p) & 1);
          if (lane == p * A + a) *row_word = w;
        }
      }
    }
  }
}

// QJL projection of the residual held in shared memory (r_s[0..d_pad)):
// lane l computes z_i for rows i = 32c + l; sign word c is the ballot of
// z_i >= 0 over the warp and is written by lane 0 to dst[c].
__device__ __forceinline__ void qjl_signs(const QParams& qp, const float* r_s, int lane,
                                          uint32_t* dst) {
  const int m = qp.m, dp = qp.d_pad;
  for (int c0 = 0; c0 < m / 32; c0 += 4) {
    float z[4] = {0.f, 0.f, 0.f, 0.f};
    const int nc = min(4, m / 32 - c0);
    for (int j = 0; j < dp; ++j) {
      const float rj = r_s[j];
      const float* st = qp.St + (size_t)j * m + (c0 * 32 + lane);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (u < nc) z[u] = fmaf(__ldg(st + u * 32), rj, z[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u < nc) {
        const uint32_t w = __ballot_sync(0xffffffffu, z[u] >= 0.0f);
        if (lane == 0) dst[c0 + u] = w;
      }
    }
  }
}

// One warp task = up to 32 consecutive vectors of one segment (= one BLOCK32
// block).  Grid-stride over tasks.
template <int A, typename T, bool PROD>
__global__ void __launch_bounds__(128) encode_hadamard_kernel(
    QParams qp, const T* __restrict__ x, int64_t ld, int64_t seg_len, int64_t seg_cap,
    int64_t blocks_per_seg, int64_t n_tasks, int layout, uint32_t* __restrict__ codes,
    uint32_t* __restrict__ signs, float* __restrict__ norms, float* __restrict__ rnorms) {
  __shared__ SmemCodebook cb;
  __shared__ float r_s[4][PROD ? 32 * A : 1];
  load_codebook(cb, qp);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const bool block_layout = layout == TQ_LAYOUT_BLOCK32;
  const int k = qp.k;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib; task < n_tasks;
       task += warps_total) {
    const int64_t s = task / blocks_per_seg;
    const int64_t b = task % blocks_per_seg;
    const int nv = (int)min64(32, seg_len - 32 * b);
    uint32_t blk[4][A];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int a = 0; a < A; ++a) blk[p][a] = 0u;
    for (int t = 0; t < nv; ++t) {
      const int64_t row = s * seg_len + 32 * b + t;
      const int64_t slot = s * seg_cap + 32 * b + t;
      const T* xr = x + row * ld;
      float v[A];
      float ss = 0.f;
#pragma unroll
      for (int a = 0; a < A; ++a) {
        const int j = 32 * a + lane;
        v[a] = j < qp.d ? to_f32(xr[j]) : 0.0f;
        ss = fmaf(v[a], v[a], ss);
      }
      ss = warp_sum(ss);
      const float n = sqrtf(ss);
      apply_signs<A>(v, qp.dmask, lane);
      warp_fwht<A>(v, lane);
      const float scale = n > 0.0f ? qp.inv_sqrt_dpad / n : 0.0f;
#pragma unroll
      for (int a = 0; a < A; ++a) v[a] *= scale;
      int idx[A];
      uint32_t row_word = 0;
      quantize_pack<A>(v, idx, cb, k, lane, &row_word, blk, t, block_layout);
      if (!block_layout && lane < k * A) codes[slot * qp.code_words + lane] = row_word;
      float nstore = n;
      if (!PROD && qp.unbiased) {  // EDEN's scale n / <y, C[idx]>
        float dot = 0.f;
#pragma unroll
        for (int a = 0; a < A; ++a) dot = fmaf(v[a], cb.c[idx[a]], dot);
        dot = warp_sum(dot);
        nstore = dot > 0.f ? n / dot : 0.f;
      }
      if (lane == 0) norms[slot] = nstore;
      if (PROD) {
        float rr = 0.f;
#pragma unroll
        for (int a = 0; a < A; ++a) {
          const float r = v[a] - cb.c[idx[a]];
          rr = fmaf(r, r, rr);
          r_s[wib][32 * a + lane] = r;
        }
        rr = warp_sum(rr);
        __syncwarp();
        qjl_signs(qp, r_s[wib], lane, signs + slot * qp.sign_words);
        if (lane == 0) put_rnorm(rnorms, slot, sqrtf(rr), qp.rnorm_f16);
        __syncwarp();
      }
    }
    if (block_layout) {
      uint32_t* dst = codes + (s * (seg_cap / 32) + b) * (int64_t)(k * 32 * A);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if (p < k)
#pragma unroll
          for (int a = 0; a < A; ++a) dst[p * 32 * A + 32 * a + lane] = blk[p][a];
    }
  }
}

// Dense path, step 1: n = ||x|| and x / n (fp32) for a chunk of vectors.
template <typename T>
__global__ void __launch_bounds__(128) normalize_rows_kernel(const T* __restrict__ x, int64_t ld,
                                                             int d, int64_t seg_len,
                                                             int64_t seg_cap, int64_t row0,
                                                             int64_t nrows,
                                                             float* __restrict__ xhat,
                                                             float* __restrict__ norms) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= nrows) return;
  const int64_t row = row0 + w;
  const T* xr = x + row * ld;
  float ss = 0.f;
  for (int j = lane; j < d; j += 32) {
    const float v = to_f32(xr[j]);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float n = sqrtf(ss);
  const float inv = n > 0.f ? 1.0f / n : 0.0f;
  for (int j = lane; j < d; j += 32) xhat[w * d + j] = to_f32(xr[j]) * inv;
  if (lane == 0) {
    const int64_t s = row / seg_len, t = row % seg_len;
    norms[s * seg_cap + t] = n;
  }
}

// Dense path, step 3: quantize rotated rows y (fp32 [nrows][d]) and pack.
// Q_prod also overwrites y with r = y - C[idx] and writes rho; the unbiased
// Q_MSE variant divides the stored norm by <y, C[idx]>.  One warp per
// 32-vector task; the host splits chunks at segment and block boundaries.
__global__ void __launch_bounds__(128) quantize_rows_kernel(
    QParams qp, float* __restrict__ y, int64_t seg_len, int64_t seg_cap, int64_t row0,
    int64_t nrows, int layout, bool prod, uint32_t* __restrict__ codes,
    float* __restrict__ norms, float* __restrict__ rnorms) {
  __shared__ SmemCodebook cb;
  load_codebook(cb, qp);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int k = qp.k, A = qp.d_pad / 32, d = qp.d;
  const int nb = (1 << k) - 1;
  const int64_t first = 32 * ((int64_t)blockIdx.x * 4 + wib);
  if (first >= nrows) return;
  const int nv = (int)min64(32, nrows - first);
  const int64_t row = row0 + first;
  const int64_t s = row / seg_len, t0 = row % seg_len;
  if (layout == TQ_LAYOUT_BLOCK32) {
    uint32_t* dst = codes + (s * (seg_cap / 32) + t0 / 32) * (int64_t)(k * 32 * A);
    for (int a = 0; a < A; ++a) {
      uint32_t blk[4] = {0u, 0u, 0u, 0u};
      for (int t = 0; t < nv; ++t) {
        const int idx = quantize_index(y[(first + t) * (int64_t)d + 32 * a + lane], cb.b, nb);
#pragma unroll
        for (int p = 0; p < 4; ++p) blk[p] |= (uint32_t)((idx >> p) & 1) << t;
      }
      for (int p = 0; p < k; ++p) dst[p * 32 * A + 32 * a + lane] = blk[p];
    }
    if (qp.unbiased && !prod) {  // EDEN's scale n / <y, C[idx]> per row
      for (int t = 0; t < nv; ++t) {
        const float* yr = y + (first + t) * (int64_t)d;
        float dot = 0.f;
        for (int a = 0; a < A; ++a) {
          const float v = yr[32 * a + lane];
          dot = fmaf(v, cb.c[quantize_index(v, cb.b, nb)], dot);
        }
        dot = warp_sum(dot);
        if (lane == 0) {
          float* nr = norms + s * seg_cap + t0 + t;
          *nr = dot > 0.f ? *nr / dot : 0.f;
        }
      }
    }
    return;
  }
  for (int t = 0; t < nv; ++t) {
    float* yr = y + (first + t) * (int64_t)d;
    const int64_t slot = s * seg_cap + t0 + t;
    float rr = 0.f, dot = 0.f;
    for (int a = 0; a < A; ++a) {
      const float v = yr[32 * a + lane];
      const int idx = quantize_index(v, cb.b, nb);
      dot = fmaf(v, cb.c[idx], dot);
      for (int p = 0; p < k; ++p) {
        const uint32_t w = __ballot_sync(0xffffffffu, (idx >> p) & 1);
        if (lane == 0) codes[slot * qp.code_words + p * A + a] = w;
      }
      if (prod) {
        const float r = v - cb.c[idx];
        rr = fmaf(r, r, rr);
        yr[32 * a + lane] = r;
      }
    }
    if (prod) {
      rr = warp_sum(rr);
      if (lane == 0) put_rnorm(rnorms, slot, sqrtf(rr), qp.rnorm_f16);
    } else if (qp.unbiased) {  // EDEN's scale n / <y, C[idx]>
      dot = warp_sum(dot);
      if (lane == 0) norms[slot] = dot > 0.f ? norms[slot] / dot : 0.f;
    }
  }
}

// Dense path, step 3 for ROW codes: one warp per row, the word positions of
// a row independent of each other so that their loads are in flight
// together (the task-per-32-rows kernel above walks them one by one).  Same
// arithmetic and order as that kernel: idx = #{B_k < y}, code word p * A + a
// = the ballot of bit p, and for Q_prod r = y - C[idx] over y with
// rho = ||r||; the unbiased Q_MSE divides the norm by <y, C[idx]>.
// With a2 given (Q_prod on the tensor-core dense path), r is written as the
// [hi | lo] fp16 operand of the S r product (hi = fp16(2^8 r), lo =
// fp16(2^8 r - hi), row stride 2 d) instead of over y.
template <int K>
__global__ void __launch_bounds__(256) quantize_rows_warp_kernel(
    QParams qp, float* __restrict__ y, int64_t seg_len, int64_t seg_cap, int64_t row0, int64_t nrows, bool prod,
    uint32_t* __restrict__ codes, float* __restrict__ norms, float* __restrict__ rnorms,
    uint16_t* __restrict__ a2) {
  __shared__ SmemCodebook cb;
  load_codebook(cb, qp);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= nrows) return;
  constexpr int k = K, nb = (1 << K) - 1;
  const int A = qp.d_pad / 32, d = qp.d;
  const int64_t row = row0 + w;
  const int64_t slot = (row / seg_len) * seg_cap + row % seg_len;
  float* yr = y + w * (int64_t)d;
  uint32_t* cw = codes + slot * qp.code_words;
  float rr = 0.f, dot = 0.f;
#pragma unroll 4
  for (int a = 0; a < A; ++a) {
    const float v = yr[32 * a + lane];
    int idx = 0;  // #{B_j < v}, as quantize_index
#pragma unroll
    for (int j = 0; j < nb; ++j) idx += (cb.b[j] < v) ? 1 : 0;
    const float c = cb.c[idx];
    dot = fmaf(v, c, dot);
#pragma unroll
    for (int p = 0; p < k; ++p) {
      const uint32_t word = __ballot_sync(0xffffffffu, (idx >> p) & 1);
      if (lane == p) cw[p * A + a] = word;
    }
    if (prod) {
      const float r = v - c;
      rr = fmaf(r, r, rr);
      if (a2) {
        const __half h = __float2half_rn(r * 256.0f);
        const __half l = __float2half_rn(r * 256.0f - __half2float(h));
        uint16_t* ar = a2 + w * (int64_t)(2 * d);
        ar[32 * a + lane] = __half_as_ushort(h);
        ar[d + 32 * a + lane] = __half_as_ushort(l);
      } else {
        yr[32 * a + lane] = r;
      }
    }
  }
  if (prod) {
    rr = warp_sum(rr);
    if (lane == 0) put_rnorm(rnorms, slot, sqrtf(rr), qp.rnorm_f16);
  } else if (qp.unbiased) {  // EDEN's scale n / <y, C[idx]>
    dot = warp_sum(dot);
    if (lane == 0) norms[slot] = dot > 0.f ? norms[slot] / dot : 0.f;
  }
}

inline void launch_quantize_rows_warp(const QParams& qp, float* y, int64_t seg_len, int64_t seg_cap, int64_t row0,
                                      int64_t nrows, bool prod, uint32_t* codes, float* norms, float* rnorms,
                                      cudaStream_t st, uint16_t* a2 = nullptr) {
  const unsigned blocks = (unsigned)ceil_div(nrows, 8);
  switch (qp.k) {
#define TQ_QRW(KK)                                                                                       \
  case KK:                                                                                              \
    quantize_rows_warp_kernel<KK><<<blocks, 256, 0, st>>>(qp, y, seg_len, seg_cap, row0, nrows, prod,  \
                                                            codes, norms, rnorms, a2);                  \
    break;
    TQ_QRW(1)
    TQ_QRW(2)
    TQ_QRW(3)
    TQ_QRW(4)
#undef TQ_QRW
    default:
      break;
  }
}

// Dense path, step 5: sign bits of z = r S^T (fp32 [nrows][m]).
__global__ void __launch_bounds__(128) pack_signs_kernel(const float* __restrict__ z, int m,
                                                         int64_t seg_len, int64_t seg_cap,
                                                         int64_t row0, int64_t nrows,
                                                         uint32_t* __restrict__ signs) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (w >= nrows) return;
  const int64_t row = row0 + w;
  const int64_t slot = (row / seg_len) * seg_cap + row % seg_len;
  for (int c = 0; c < m / 32; ++c) {
    const uint32_t word = __ballot_sync(0xffffffffu, z[w * m + 32 * c + lane] >= 0.0f);
    if (lane == 0) signs[slot * (m / 32) + c] = word;
  }
}

}  // namespace tq
