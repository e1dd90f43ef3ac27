// Query preparation, inner-product scores, top-k and decode.
//
// Score estimator (TurboQuant blog notes, unbiased inner-product estimator
// with the residual norm; explainer §8 QJL decoder; turboquant-pytorch
// inner_product / asymmetric_attention_scores):
//   q' = Pi q, u = S q'   (once per query)
//   s = n ( <q', C[idx]> + kappa rho <u, 2 sigma - 1> ),  kappa = sqrt(pi/2)/m
#pragma once

#include "tq_device.cuh"
#include "tq_encode.cuh"

namespace tq {

// q' = Pi pad(q) and u = S q' for QPB queries per block of 128 or 256
// threads: warp w < QPB rotates query w (register FWHT), then every thread
// forms outputs of u, each a sum over j in ascending order with coalesced
// loads of S^T (shared by the block's queries), 32 loads in flight.
template <int A, int QPB>
__global__ void __launch_bounds__(256) query_prep_hadamard_kernel(QParams qp,
                                                                  const float* __restrict__ q,
                                                                  int64_t nq, int64_t ldq,
                                                                  float* __restrict__ qrot,
                                                                  float* __restrict__ u) {
  __shared__ float qs[QPB][32 * A];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t q0 = (int64_t)blockIdx.x * QPB;
  if (wib < QPB && q0 + wib < nq) {
    const int64_t w = q0 + wib;
    float v[A];
#pragma unroll
    for (int a = 0; a < A; ++a) {
      const int j = 32 * a + lane;
      v[a] = j < qp.d ? q[w * ldq + j] : 0.f;
    }
    apply_signs<A>(v, qp.dmask, lane);
    warp_fwht<A>(v, lane);
#pragma unroll
    for (int a = 0; a < A; ++a) {
      v[a] *= qp.inv_sqrt_dpad;
      qrot[w * qp.d_pad + 32 * a + lane] = v[a];
      qs[wib][32 * a + lane] = v[a];
    }
  }
  __syncthreads();
  if (!u) return;
  for (int i = threadIdx.x; i < qp.m; i += blockDim.x) {
    float acc[QPB];
#pragma unroll
    for (int t = 0; t < QPB; ++t) acc[t] = 0.f;
#pragma unroll 32
    for (int j = 0; j < qp.d_pad; ++j) {
      const float sv = __ldg(qp.St + (size_t)j * qp.m + i);
#pragma unroll
      for (int t = 0; t < QPB; ++t) acc[t] = fmaf(sv, qs[t][j], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < QPB; ++t)
      if (q0 + t < nq) u[(q0 + t) * qp.m + i] = acc[t];
  }
}

// scores[a][t] for a tile of QT queries (q' and u staged in shared memory)
// and 128 vectors per CTA (one thread per vector).
constexpr int kScoreThreads = 128;

__global__ void __launch_bounds__(kScoreThreads) scores_kernel(
    QParams qp, const float* __restrict__ qrot, const float* __restrict__ u, int64_t nq, int qt,
    const uint32_t* __restrict__ codes, const uint32_t* __restrict__ signs,
    const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n_vec,
    float* __restrict__ scores) {
  extern __shared__ float dyn[];
  __shared__ SmemCodebook cb;
  load_codebook(cb, qp);
  const int dp = qp.d_pad, m = qp.m, k = qp.k;
  const int wpp = dp / 32;
  const int64_t q0 = (int64_t)blockIdx.y * qt;
  const int nql = (int)min64(qt, nq - q0);
  float* qs = dyn;                 // [qt][dp]
  float* us = dyn + (size_t)qt * dp;  // [qt][m]
  for (int e = threadIdx.x; e < nql * dp; e += blockDim.x) qs[e] = qrot[q0 * dp + e];
  for (int e = threadIdx.x; e < nql * m; e += blockDim.x) us[e] = u[q0 * m + e];
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_vec) return;
  constexpr int kMaxQT = 32;
  float am[kMaxQT], aq[kMaxQT];
#pragma unroll
  for (int a = 0; a < kMaxQT; ++a) am[a] = aq[a] = 0.f;
  const uint32_t* cw = codes + t * qp.code_words;
  for (int w = 0; w < wpp; ++w) {
    uint32_t pw[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) pw[p] = p < k ? cw[p * wpp + w] : 0u;
    for (int i = 0; i < 32; ++i) {
      int idx = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) idx |= (int)((pw[p] >> i) & 1u) << p;
      const float c = cb.c[idx];
      const int j = 32 * w + i;
#pragma unroll
      for (int a = 0; a < kMaxQT; ++a)
        if (a < nql) am[a] = fmaf(qs[a * dp + j], c, am[a]);
    }
  }
  if (m > 0) {
    const uint32_t* sw = signs + t * qp.sign_words;
    for (int w = 0; w < m / 32; ++w) {
      const uint32_t word = sw[w];
      for (int i = 0; i < 32; ++i) {
        const float sg = ((word >> i) & 1u) ? 1.0f : -1.0f;
        const int j = 32 * w + i;
#pragma unroll
        for (int a = 0; a < kMaxQT; ++a)
          if (a < nql) aq[a] = fmaf(us[a * m + j], sg, aq[a]);
      }
    }
  }
  const float n = norms[t];
  const float kr = m > 0 ? qp.kappa * get_rnorm(rnorms, t, qp.rnorm_f16) : 0.f;
#pragma unroll
  for (int a = 0; a < kMaxQT; ++a)
    if (a < nql) scores[(q0 + a) * n_vec + t] = n * (am[a] + kr * aq[a]);
}

// Top-k per row of a score matrix: (score desc, index asc).  One CTA per row;
// every thread keeps a sorted list of its best K candidates, then K rounds of
// a block-wide arg-max pick the winners.
constexpr int kTopkMax = 32;
constexpr int kTopkThreads = 256;

__device__ __forceinline__ bool better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores,
                                                            int64_t n_vec, int K,
                                                            float* __restrict__ top_s,
                                                            int64_t* __restrict__ top_i) {
  __shared__ float ws_s[kTopkThreads / 32];
  __shared__ int64_t ws_i[kTopkThreads / 32];
  __shared__ int ws_t[kTopkThreads / 32];
  __shared__ int winner;
  const int64_t row = blockIdx.x;
  const float* s = scores + row * n_vec;
  float ls[kTopkMax];
  int64_t li[kTopkMax];
  int cnt = 0;
  for (int64_t i = threadIdx.x; i < n_vec; i += blockDim.x) {
    const float v = s[i];
    if (cnt == K && !better(v, i, ls[K - 1], li[K - 1])) continue;
    int pos = cnt < K ? cnt : K - 1;
    if (cnt < K) ++cnt;
    while (pos > 0 && better(v, i, ls[pos - 1], li[pos - 1])) {
      ls[pos] = ls[pos - 1];
      li[pos] = li[pos - 1];
      --pos;
    }
    ls[pos] = v;
    li[pos] = i;
  }
  int head = 0;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int r = 0; r < K; ++r) {
    float bs = head < cnt ? ls[head] : -INFINITY;
    int64_t bi = head < cnt ? li[head] : INT64_MAX;
    int bt = threadIdx.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const int ot = __shfl_xor_sync(0xffffffffu, bt, o);
      if (better(os, oi, bs, bi)) {
        bs = os;
        bi = oi;
        bt = ot;
      }
    }
    if (lane == 0) {
      ws_s[wid] = bs;
      ws_i[wid] = bi;
      ws_t[wid] = bt;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int best = 0;
      for (int w = 1; w < kTopkThreads / 32; ++w)
        if (better(ws_s[w], ws_i[w], ws_s[best], ws_i[best])) best = w;
      top_s[row * K + r] = ws_s[best];
      top_i[row * K + r] = ws_i[best] == INT64_MAX ? -1 : ws_i[best];
      winner = ws_t[best];
    }
    __syncthreads();
    if (threadIdx.x == winner) ++head;
    __syncthreads();
  }
}

// Decode: x~ = n Pi^T (C[idx] [+ kappa rho S^T (2 sigma - 1)]), one warp per
// vector.  Hadamard: Pi^T y = D H y / sqrt(d_pad).
template <int A>
__global__ void __launch_bounds__(128) decode_hadamard_kernel(
    QParams qp, int layout, const uint32_t* __restrict__ codes,
    const uint32_t* __restrict__ signs, const float* __restrict__ norms,
    const float* __restrict__ rnorms, int64_t n_vec, int64_t seg_len, int64_t seg_cap,
    float* __restrict__ out, int64_t ldo) {
  __shared__ SmemCodebook cb;
  load_codebook(cb, qp);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (w >= n_vec) return;
  const int64_t s = w / seg_len, t = w % seg_len;
  const int64_t slot = s * seg_cap + t;
  const int k = qp.k;
  float v[A];
#pragma unroll
  for (int a = 0; a < A; ++a) {
    int idx = 0;
    for (int p = 0; p < k; ++p) {
      uint32_t word;
      if (layout == TQ_LAYOUT_BLOCK32)
        word = codes[(s * (seg_cap / 32) + t / 32) * (int64_t)(k * 32 * A) + p * 32 * A + 32 * a + lane] >> (t % 32);
      else
        word = codes[slot * qp.code_words + p * A + a] >> lane;
      idx |= (int)(word & 1u) << p;
    }
    v[a] = cb.c[idx];
  }
  if (signs && qp.m > 0) {
    const float kr = qp.kappa * get_rnorm(rnorms, slot, qp.rnorm_f16);
    const uint32_t* sw = signs + slot * qp.sign_words;
#pragma unroll
    for (int a = 0; a < A; ++a) {
      float acc = 0.f;
      const int j = 32 * a + lane;
      for (int i = 0; i < qp.m; ++i) {
        const float sg = ((sw[i / 32] >> (i % 32)) & 1u) ? 1.f : -1.f;
        acc = fmaf(__ldg(qp.S + (size_t)i * qp.d_pad + j), sg, acc);
      }
      v[a] = fmaf(kr, acc, v[a]);
    }
  }
  warp_fwht<A>(v, lane);
  apply_signs<A>(v, qp.dmask, lane);
  const float sc = norms[slot] * qp.inv_sqrt_dpad;
#pragma unroll
  for (int a = 0; a < A; ++a) {
    const int j = 32 * a + lane;
    if (j < qp.d) out[w * ldo + j] = v[a] * sc;
  }
}

// Dense-rotation decode (one warp per vector, rotated vector in shared memory).
__global__ void __launch_bounds__(128) decode_dense_kernel(
    QParams qp, int layout, const uint32_t* __restrict__ codes,
    const uint32_t* __restrict__ signs, const float* __restrict__ norms,
    const float* __restrict__ rnorms, int64_t n_vec, int64_t seg_len, int64_t seg_cap,
    float* __restrict__ out, int64_t ldo) {
  extern __shared__ float dyn[];
  __shared__ SmemCodebook cb;
  load_codebook(cb, qp);
  __syncthreads();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t w = (int64_t)blockIdx.x * 4 + wib;
  if (w >= n_vec) return;
  const int d = qp.d, A = d / 32, k = qp.k;
  float* ys = dyn + wib * d;
  const int64_t s = w / seg_len, t = w % seg_len;
  const int64_t slot = s * seg_cap + t;
  for (int a = 0; a < A; ++a) {
    int idx = 0;
    for (int p = 0; p < k; ++p) {
      uint32_t word;
      if (layout == TQ_LAYOUT_BLOCK32)
        word = codes[(s * (seg_cap / 32) + t / 32) * (int64_t)(k * 32 * A) + p * 32 * A + 32 * a + lane] >> (t % 32);
      else
        word = codes[slot * qp.code_words + p * A + a] >> lane;
      idx |= (int)(word & 1u) << p;
    }
    float v = cb.c[idx];
    if (signs && qp.m > 0) {
      const uint32_t* sw = signs + slot * qp.sign_words;
      float acc = 0.f;
      const int j = 32 * a + lane;
      for (int i = 0; i < qp.m; ++i) {
        const float sg = ((sw[i / 32] >> (i % 32)) & 1u) ? 1.f : -1.f;
        acc = fmaf(__ldg(qp.S + (size_t)i * d + j), sg, acc);
      }
      v = fmaf(qp.kappa * get_rnorm(rnorms, slot, qp.rnorm_f16), acc, v);
    }
    ys[32 * a + lane] = v;
  }
  __syncwarp();
  const float n = norms[slot];
  for (int i = lane; i < d; i += 32) {
    float acc = 0.f;
    for (int j = 0; j < d; ++j) acc = fmaf(__ldg(qp.Pi + (size_t)j * d + i), ys[j], acc);
    out[w * ldo + i] = acc * n;
  }
}

}  // namespace tq
