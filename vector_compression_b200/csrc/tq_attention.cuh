// Fused decode attention over a compressed KV cache (turboquant-pytorch
// Pattern 1: scores from compressed keys, softmax, weighted sum of the
// Q_MSE-reconstructed values), split over sequence chunks.
//
// Per (layer, batch, kv-head) group and chunk, for each of the G query heads
// sharing the KV head:
//   s_t   = n_t ( <q', C_K[idx_t]> + kappa rho_t <u, 2 sigma_t - 1> )
//   online softmax of alpha s_t (running max m and sum l)
//   o_rot = sum_t p_t ||v_t|| C_V[iv_t]       (rotated value domain)
// and a combine kernel merges the chunks by log-sum-exp and applies Pi_V^T
// once per output vector (Pi^T is linear, so averaging before the inverse
// rotation equals rotating every value first).
#pragma once

#include "tq_device.cuh"
#include "tq_encode.cuh"

namespace tq {

constexpr int kAttnThreads = 128;
constexpr int kAttnMaxG = 16;

struct AttnShape {
  int G;             // query heads per KV head
  int groups;        // L * B * Hkv
  int n_chunks;
  int chunk;         // tokens per chunk (multiple of 32)
  int64_t seq, cap;
  float scale;
};

// Partial results per (group, chunk, head): m, l, o[d_pad].
__device__ __forceinline__ float* partial_ptr(float* part, int d_pad, int G, int n_chunks,
                                              int g, int c, int h) {
  return part + (((int64_t)g * n_chunks + c) * G + h) * (int64_t)(d_pad + 2);
}

template <int NC>  // value coordinates per thread: d_pad <= 128 * NC
__global__ void __launch_bounds__(kAttnThreads) attention_chunk_kernel(
    QParams kp, QParams vp, AttnShape sh, const float* __restrict__ qrot,
    const float* __restrict__ u, const uint32_t* __restrict__ kcodes,
    const uint32_t* __restrict__ ksigns, const float* __restrict__ knorms,
    const float* __restrict__ krnorms, const uint32_t* __restrict__ vcodes,
    const float* __restrict__ vnorms, float* __restrict__ part) {
  extern __shared__ float dyn[];
  __shared__ SmemCodebook kcb, vcb;
  __shared__ float p_s[32][kAttnMaxG];
  __shared__ float corr_s[kAttnMaxG];
  __shared__ float m_s[kAttnMaxG], l_s[kAttnMaxG];
  const int G = sh.G;
  const int dp = kp.d_pad, m = kp.m, kk = kp.k, kv = vp.k;
  const int g = blockIdx.y, c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  float* qs = dyn;                      // [G][dp]
  float* us = dyn + (size_t)G * dp;     // [G][m]
  if (tid < kMaxLevels) {
    kcb.c[tid] = kp.centroids[tid];
    kcb.b[tid] = kp.boundaries[tid];
    vcb.c[tid] = vp.centroids[tid];
    vcb.b[tid] = vp.boundaries[tid];
  }
  for (int e = tid; e < G * dp; e += blockDim.x) qs[e] = qrot[(int64_t)g * G * dp + e];
  for (int e = tid; e < G * m; e += blockDim.x) us[e] = u[(int64_t)g * G * m + e];
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  __syncthreads();

  const int64_t t_begin = (int64_t)c * sh.chunk;
  const int64_t t_end = min64(sh.seq, t_begin + sh.chunk);
  const int64_t kbase = (int64_t)g * sh.cap;           // key rows of this group
  const int64_t vblk0 = (int64_t)g * (sh.cap / 32);     // value blocks of this group
  const int wpp = dp / 32;

  float o[kAttnMaxG][NC];
#pragma unroll
  for (int h = 0; h < kAttnMaxG; ++h)
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) o[h][cc] = 0.f;

  for (int64_t tb = t_begin; tb < t_end; tb += 32) {
    // ---- scores: warp wid handles heads wid, wid+4, ...; lane = token
    const int64_t t = tb + lane;
    const bool valid = t < t_end;
    constexpr int HW = kAttnMaxG / 4;
    float am[HW], aq[HW];
#pragma unroll
    for (int i = 0; i < HW; ++i) am[i] = aq[i] = 0.f;
    float kn = 0.f, kr = 0.f;
    if (valid) {
      const uint32_t* cw = kcodes + (kbase + t) * kp.code_words;
      for (int w = 0; w < wpp; ++w) {
        uint32_t pw[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) pw[p] = p < kk ? cw[p * wpp + w] : 0u;
        for (int i = 0; i < 32; ++i) {
          int idx = 0;
#pragma unroll
          for (int p = 0; p < 4; ++p) idx |= (int)((pw[p] >> i) & 1u) << p;
          const float cval = kcb.c[idx];
          const int j = 32 * w + i;
#pragma unroll
          for (int hh = 0; hh < HW; ++hh) {
            const int h = wid + 4 * hh;
            if (h < G) am[hh] = fmaf(qs[h * dp + j], cval, am[hh]);
          }
        }
      }
      const uint32_t* sw = ksigns + (kbase + t) * kp.sign_words;
      for (int w = 0; w < m / 32; ++w) {
        const uint32_t word = sw[w];
        for (int i = 0; i < 32; ++i) {
          const float sg = ((word >> i) & 1u) ? 1.f : -1.f;
          const int j = 32 * w + i;
#pragma unroll
          for (int hh = 0; hh < HW; ++hh) {
            const int h = wid + 4 * hh;
            if (h < G) aq[hh] = fmaf(us[h * m + j], sg, aq[hh]);
          }
        }
      }
      kn = knorms[kbase + t];
      kr = kp.kappa * get_rnorm(krnorms, kbase + t, kp.rnorm_f16);
    }
    const float vn = valid ? vnorms[kbase + t] : 0.f;
#pragma unroll
    for (int hh = 0; hh < HW; ++hh) {
      const int h = wid + 4 * hh;
      if (h < G) {
        const float x = valid ? sh.scale * (kn * (am[hh] + kr * aq[hh])) : -INFINITY;
        const float m_old = m_s[h];
        const float m_new = fmaxf(m_old, warp_max(x));
        float p = 0.f, corr = 1.f;
        if (m_new != -INFINITY) {
          p = valid ? expf(x - m_new) : 0.f;
          corr = expf(m_old - m_new);
        }
        const float psum = warp_sum(p);
        p_s[lane][h] = p * vn;
        if (lane == 0) {
          corr_s[h] = corr;
          m_s[h] = m_new;
          l_s[h] = l_s[h] * corr + psum;
        }
      }
    }
    __syncthreads();
    // ---- values: thread tid owns coordinates tid + 128 cc
    const int nt = (int)min64(32, t_end - tb);
    const uint32_t* vb = vcodes + (vblk0 + tb / 32) * (int64_t)(kv * dp);
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) {
      const int j = tid + 128 * cc;
      if (j >= dp) continue;
      uint32_t pw[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) pw[p] = p < kv ? vb[p * dp + j] : 0u;
#pragma unroll
      for (int h = 0; h < kAttnMaxG; ++h)
        if (h < G) o[h][cc] *= corr_s[h];
      for (int i = 0; i < nt; ++i) {
        int idx = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) idx |= (int)((pw[p] >> i) & 1u) << p;
        const float cval = vcb.c[idx];
#pragma unroll
        for (int h = 0; h < kAttnMaxG; ++h)
          if (h < G) o[h][cc] = fmaf(p_s[i][h], cval, o[h][cc]);
      }
    }
    __syncthreads();
  }
  // ---- partials
  for (int h = 0; h < G; ++h) {
    float* pp = partial_ptr(part, dp, G, sh.n_chunks, g, c, h);
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) {
      const int j = tid + 128 * cc;
      if (j < dp) pp[2 + j] = o[h][cc];
    }
    if (tid == 0) {
      pp[0] = m_s[h];
      pp[1] = l_s[h];
    }
  }
}

// Merge chunk partials by log-sum-exp and apply Pi_V^T (Hadamard: D H / sqrt(d_pad)).
// One block of eight warps per (group, head): the running maximum over the
// chunks is a block reduction, warp w sums the chunks c = w mod 8, and warp 0
// adds the eight partial sums in warp order, then rotates and stores.
template <int A>
__global__ void __launch_bounds__(256) attention_combine_hadamard_kernel(
    QParams vp, AttnShape sh, const float* __restrict__ part, float* __restrict__ out,
    int Hq, int Hkv) {
  constexpr int kW = 8;
  __shared__ float sm[kW], sl[kW];
  __shared__ float sv[kW][32 * A];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t w = blockIdx.x;  // (group, head)
  const int g = (int)(w / sh.G), h = (int)(w % sh.G);
  const int dp = vp.d_pad;
  float M = -INFINITY;
  for (int c = threadIdx.x; c < sh.n_chunks; c += 32 * kW)
    M = fmaxf(M, partial_ptr((float*)part, dp, sh.G, sh.n_chunks, g, c, h)[0]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) sm[wib] = M;
  __syncthreads();
  M = sm[0];
#pragma unroll
  for (int i = 1; i < kW; ++i) M = fmaxf(M, sm[i]);
  float L = 0.f;
  float v[A];
#pragma unroll
  for (int a = 0; a < A; ++a) v[a] = 0.f;
  for (int c = wib; c < sh.n_chunks; c += kW) {
    const float* pp = partial_ptr((float*)part, dp, sh.G, sh.n_chunks, g, c, h);
    if (pp[0] == -INFINITY) continue;
    const float e = expf(pp[0] - M);
    L = fmaf(e, pp[1], L);
#pragma unroll
    for (int a = 0; a < A; ++a) v[a] = fmaf(e, pp[2 + 32 * a + lane], v[a]);
  }
  if (lane == 0) sl[wib] = L;
#pragma unroll
  for (int a = 0; a < A; ++a) sv[wib][32 * a + lane] = v[a];
  __syncthreads();
  if (wib != 0) return;
  L = sl[0];
#pragma unroll
  for (int i = 1; i < kW; ++i) L += sl[i];
#pragma unroll
  for (int a = 0; a < A; ++a) {
    float t = sv[0][32 * a + lane];
#pragma unroll
    for (int i = 1; i < kW; ++i) t += sv[i][32 * a + lane];
    v[a] = t;
  }
  const float inv = L > 0.f ? 1.0f / L : 0.f;
  warp_fwht<A>(v, lane);
  apply_signs<A>(v, vp.dmask, lane);
  const float sc = inv * vp.inv_sqrt_dpad;
  // group g = (l * B + b) * Hkv + kvh; query head = kvh * G + h
  const int64_t lb = g / Hkv;
  const int kvh = g % Hkv;
  float* o = out + (lb * Hq + (int64_t)kvh * sh.G + h) * vp.d;
#pragma unroll
  for (int a = 0; a < A; ++a) {
    const int j = 32 * a + lane;
    if (j < vp.d) o[j] = v[a] * sc;
  }
}

}  // namespace tq
