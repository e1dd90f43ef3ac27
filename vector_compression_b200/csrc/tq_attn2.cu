// Decode attention over a compressed KV cache on the tensor cores
// (turboquant-pytorch Pattern 1: scores from compressed keys, softmax,
// weighted sum of the Q_MSE-reconstructed values; TurboQuant blog notes,
// Q_prod estimator; explainer §8).
//
// Exact bit features.  A symmetric 2^k-level codebook is an odd function of
// the index bits u_p = 2 b_p - 1, so C[idx] = sum over odd subsets S of
// alpha_S prod_{p in S} u_p, and prod_{p in S} u_p = 2 b_S - 1 with
// b_S = XOR_{p in S} b_p.  Hence
//   <q', C[idx]>          = sum_S alpha_S (2 <q', b_S> - sum q'),
//   <u, 2 sigma - 1>      = 2 <u, sigma> - sum u,
//   sum_t w_t C[idx_t]_j  = sum_S alpha_S (2 sum_t w_t b_S,tj - sum_t w_t):
// every contraction is against 0/1 bit matrices, which are exact in fp16.
// Bits become fp16 {0, 2.0} with one rotate and one AND per pair.  The query
// side (alpha_S q', u) and the softmax weights are split into fp16 hi + lo
// parts (as columns of the N = 8 tile for up to 4 query heads per KV head,
// as a second n-tile for 5..8 heads), so they carry ~22 significant bits.
//
// Per CTA: one (layer, batch, kv-head) group and one chunk of tokens, 4
// warps.  Tokens go in super-blocks of 64 (two 32-token value blocks).  Warp v
// scores 16 tokens of the super-block with m16n8k16 MMAs (rows = tokens,
// K = bit features, N = heads x {hi, lo}); the block maxima
// are exchanged through shared memory, the weights are formed, transposed
// into B-operand order with movmatrix and shared; then every warp
// accumulates all 64 tokens into its 32 value coordinates (rows = value
// coordinate features, K = tokens, N = 8).  Partial (m, l, o_rot) per chunk
// go to the workspace; the combine kernel merges chunks and applies Pi_V^T.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_attn2.h"
#include "tq_device.cuh"

namespace tq {
namespace attn2 {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int DP = 128;      // rotated dimension of this kernel
constexpr int WPP = DP / 32; // words per code plane
constexpr int M = 128;       // QJL rows

__device__ __forceinline__ uint32_t feat2(uint32_t w, int q) {
  // bits q and q + 16 of w -> fp16 pair {0 or 2.0, 0 or 2.0} (bit 14 / 30)
  const uint32_t r = __funnelshift_l(w, w, (uint32_t)(14 - q) & 31u);
  return r & 0x40004000u;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t h2pack(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float hhi(float x) { return __half2float(__float2half_rn(x)); }

// Number of odd-subset features of a k-bit code: 2^(k-1).
template <int K>
struct NF {
  static constexpr int v = 1 << (K - 1);
};

// Feature word S of one coordinate block from the k plane words p[0..k):
// odd subsets in the order {0},{1},...,{k-1}, then the triples.
template <int K>
__device__ __forceinline__ uint32_t feature_word(const uint32_t* p, int f) {
  if (f < K) return p[f];
  // triples (k = 3: {0,1,2}; k = 4: {0,1,2},{0,1,3},{0,2,3},{1,2,3})
  const int t = f - K;
  if (K == 3) return p[0] ^ p[1] ^ p[2];
  const int skip = 3 - t;  // the element left out of the 4-set
  uint32_t x = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q != skip) x ^= p[q];
  return x;
}

// token index (within a 32-token value block) of score row r of the 16-token
// half `half`: K-column r of the value MMA reads bit (8 half + 4 (r/8) +
// (r%8)/2 + 16 (r%2)) of a value word.
__device__ __forceinline__ int tok_of_row(int half, int r) {
  return 8 * half + 4 * (r >> 3) + ((r & 7) >> 1) + 16 * (r & 1);
}

template <int KK, int KV, bool HL>
__global__ void __launch_bounds__(kThreads) attn_chunk_kernel(Params P) {
  constexpr int FK = NF<KK>::v;           // key code features per coordinate
  constexpr int FV = NF<KV>::v;           // value code features per coordinate
  constexpr int KW = KK * WPP;            // key code words per token
  constexpr int SW = M / 32;              // sign words per token
  constexpr int KSTEP_C = FK * WPP * 2;   // k-steps over key code features
  constexpr int KSTEP_S = SW * 2;         // k-steps over signs
  constexpr int MT = FV * 2;              // value m-tiles per warp (32 coordinates)

  __shared__ float s_bmax[kWarps][8];
  __shared__ float s_psum[kWarps][8];
  __shared__ float s_wsum[kWarps][8];
  __shared__ uint4 s_pb[kWarps][32];  // B fragments: hi (x, y), lo (z, w) n-tiles
  __shared__ float s_cm[8], s_cq[8];
  __shared__ float s_qc[8][DP];
  __shared__ float s_u[8][M];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int G = P.G;
  const int grp = blockIdx.y, chunk = blockIdx.x;

  // ---- query side: q' and u of the G heads (from the query-prep kernel)
  for (int e = tid; e < G * DP; e += kThreads) s_qc[e / DP][e % DP] = P.qrot[(int64_t)grp * G * DP + e];
  for (int e = tid; e < G * M; e += kThreads) s_u[e / M][e % M] = P.u[(int64_t)grp * G * M + e];
  __syncthreads();
  if (tid < G) {
    float sq = 0.f, su = 0.f;
    for (int j = 0; j < DP; ++j) sq += s_qc[tid][j];
    for (int i = 0; i < M; ++i) su += s_u[tid][i];
    s_cm[tid] = -P.kalpha_sum * sq;
    s_cq[tid] = -su;
  }
  // B fragments of the score MMA, column n = g.  HL (G <= 4): head g/2, hi
  // part for even g, lo part for odd g.  Otherwise head g: hi parts in bq,
  // lo parts in bql (a second n-tile), so every query coefficient carries
  // ~22 significant bits.
  const int hn = HL ? (g >> 1) : g;
  const bool hlo = HL && (g & 1);
  const bool col_ok = hn < G;
  uint32_t bq[KSTEP_C + KSTEP_S][2];
  uint32_t bql[HL ? 1 : KSTEP_C + KSTEP_S][2];
#pragma unroll
  for (int kb = 0; kb < KSTEP_C + KSTEP_S; ++kb) {
    const int w = kb >> 1, half = kb & 1;
    float v[4], vl[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // pair slots: (q, q+16) with q = 8 half + c (i = 0,1) and q = 8 half + 4 + c (i = 2,3)
      const int q = 8 * half + (i >= 2 ? 4 : 0) + c + ((i & 1) ? 16 : 0);
      float x = 0.f;
      if (col_ok) {
        if (kb < KSTEP_C) {
          const int f = w / WPP, j = 32 * (w % WPP) + q;
          x = P.kalpha[f] * s_qc[hn][j];
        } else {
          const int i2 = 32 * (w - FK * WPP) + q;
          x = s_u[hn][i2];
        }
      }
      const float h = hhi(x);
      v[i] = HL ? (hlo ? x - h : h) : h;
      vl[i] = x - h;
    }
    bq[kb][0] = h2pack(v[0], v[1]);
    bq[kb][1] = h2pack(v[2], v[3]);
    if (!HL) {
      bql[HL ? 0 : kb][0] = h2pack(vl[0], vl[1]);
      bql[HL ? 0 : kb][1] = h2pack(vl[2], vl[3]);
    }
  }
  __syncthreads();

  // per-thread softmax state for the heads of this thread's accumulator columns
  // (columns 2c, 2c+1): HL -> head c (hi, lo); else heads 2c, 2c+1
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, w_run[2] = {0.f, 0.f};
  float acc[MT][4];
  float accl[HL ? 1 : MT][4];  // G > 4: accumulators of the lo weight parts
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll
  for (int i = 0; i < (HL ? 1 : MT); ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) accl[i][j] = 0.f;

  const int64_t t_begin = (int64_t)chunk * P.chunk;
  const int64_t t_end = min64(P.seq, t_begin + P.chunk);
  const int64_t krow0 = (int64_t)grp * P.cap;
  const int64_t vblk0 = (int64_t)grp * (P.cap / 32);
  const float kappa = P.kappa;
  const float scale = P.scale;

  for (int64_t sb = t_begin; sb < t_end; sb += 64) {
    // ================= producer: scores of tokens of block `warp`
    const int vb = warp >> 1, half = warp & 1;
    const int r1 = g, r2 = g + 8;
    const int64_t T1 = sb + 32 * vb + tok_of_row(half, r1);
    const int64_t T2 = sb + 32 * vb + tok_of_row(half, r2);
    const bool ok1 = T1 < t_end, ok2 = T2 < t_end;
    uint32_t k1[KW + SW], k2[KW + SW];
    {
      const uint32_t* p1 = P.kcodes + (krow0 + T1) * KW;
      const uint32_t* p2 = P.kcodes + (krow0 + T2) * KW;
#pragma unroll
      for (int i = 0; i < KW; i += 4) {
        const uint4 a = ok1 ? *reinterpret_cast<const uint4*>(p1 + i) : make_uint4(0, 0, 0, 0);
        const uint4 b = ok2 ? *reinterpret_cast<const uint4*>(p2 + i) : make_uint4(0, 0, 0, 0);
        k1[i] = a.x; k1[i + 1] = a.y; k1[i + 2] = a.z; k1[i + 3] = a.w;
        k2[i] = b.x; k2[i + 1] = b.y; k2[i + 2] = b.z; k2[i + 3] = b.w;
      }
      const uint32_t* s1 = P.ksigns + (krow0 + T1) * SW;
      const uint32_t* s2 = P.ksigns + (krow0 + T2) * SW;
#pragma unroll
      for (int i = 0; i < SW; i += 4) {
        const uint4 a = ok1 ? *reinterpret_cast<const uint4*>(s1 + i) : make_uint4(0, 0, 0, 0);
        const uint4 b = ok2 ? *reinterpret_cast<const uint4*>(s2 + i) : make_uint4(0, 0, 0, 0);
        k1[KW + i] = a.x; k1[KW + i + 1] = a.y; k1[KW + i + 2] = a.z; k1[KW + i + 3] = a.w;
        k2[KW + i] = b.x; k2[KW + i + 1] = b.y; k2[KW + i + 2] = b.z; k2[KW + i + 3] = b.w;
      }
    }
    const float n1 = ok1 ? P.knorms[krow0 + T1] : 0.f, n2 = ok2 ? P.knorms[krow0 + T2] : 0.f;
    const float kr1 = ok1 ? kappa * get_rnorm(P.krnorms, krow0 + T1, P.kr16) : 0.f;
    const float kr2 = ok2 ? kappa * get_rnorm(P.krnorms, krow0 + T2, P.kr16) : 0.f;
    const float vn1 = ok1 ? P.vnorms[krow0 + T1] : 0.f, vn2 = ok2 ? P.vnorms[krow0 + T2] : 0.f;

    float am[4] = {0.f, 0.f, 0.f, 0.f}, aq[4] = {0.f, 0.f, 0.f, 0.f};
    float aml[4] = {0.f, 0.f, 0.f, 0.f}, aql[4] = {0.f, 0.f, 0.f, 0.f};  // lo n-tile (G > 4)
    // key code features: word index w = f * WPP + cw over feature planes
#pragma unroll
    for (int f = 0; f < FK; ++f) {
#pragma unroll
      for (int cw = 0; cw < WPP; ++cw) {
        uint32_t pl1[KK], pl2[KK];
#pragma unroll
        for (int p = 0; p < KK; ++p) {
          pl1[p] = k1[p * WPP + cw];
          pl2[p] = k2[p * WPP + cw];
        }
        const uint32_t W1 = feature_word<KK>(pl1, f), W2 = feature_word<KK>(pl2, f);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int kb = 2 * (f * WPP + cw) + hh;
          const int q0 = 8 * hh + c, q1 = 8 * hh + 4 + c;
          const uint32_t a0 = feat2(W1, q0), a1 = feat2(W2, q0), a2 = feat2(W1, q1), a3 = feat2(W2, q1);
          mma16816(am, a0, a1, a2, a3, bq[kb][0], bq[kb][1]);
          if (!HL) mma16816(aml, a0, a1, a2, a3, bql[HL ? 0 : kb][0], bql[HL ? 0 : kb][1]);
        }
      }
    }
#pragma unroll
    for (int sw = 0; sw < SW; ++sw) {
      const uint32_t W1 = k1[KW + sw], W2 = k2[KW + sw];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int kb = KSTEP_C + 2 * sw + hh;
        const int q0 = 8 * hh + c, q1 = 8 * hh + 4 + c;
        const uint32_t a0 = feat2(W1, q0), a1 = feat2(W2, q0), a2 = feat2(W1, q1), a3 = feat2(W2, q1);
        mma16816(aq, a0, a1, a2, a3, bq[kb][0], bq[kb][1]);
        if (!HL) mma16816(aql, a0, a1, a2, a3, bql[HL ? 0 : kb][0], bql[HL ? 0 : kb][1]);
      }
    }
    // scores x = scale * n (mse + C_m + kappa rho (qjl + C_q)) per row and head slot
    float x[2][2];  // [row (g, g+8)][head slot]
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      const int h = HL ? c : 2 * c + hs;
      const bool hv = h < G && (!HL || hs == 0);
      float mse1, qjl1, mse2, qjl2;
      if (HL) {
        mse1 = am[0] + am[1];
        qjl1 = aq[0] + aq[1];
        mse2 = am[2] + am[3];
        qjl2 = aq[2] + aq[3];
      } else {
        mse1 = am[hs] + aml[hs];
        qjl1 = aq[hs] + aql[hs];
        mse2 = am[2 + hs] + aml[2 + hs];
        qjl2 = aq[2 + hs] + aql[2 + hs];
      }
      const float cm = hv ? s_cm[h] : 0.f, cq = hv ? s_cq[h] : 0.f;
      x[0][hs] = (hv && ok1) ? scale * n1 * (mse1 + cm + kr1 * (qjl1 + cq)) : -INFINITY;
      x[1][hs] = (hv && ok2) ? scale * n2 * (mse2 + cm + kr2 * (qjl2 + cq)) : -INFINITY;
    }
    // block max per head slot over the 16 rows (reduce over g: lanes xor 4, 8, 16)
    float bm[2];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      float v = fmaxf(x[0][hs], x[1][hs]);
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      bm[hs] = v;
    }
    if (g == 0) {
      s_bmax[warp][2 * c] = bm[0];
      s_bmax[warp][2 * c + 1] = bm[1];
    }
    __syncthreads();
    // new running max (same on every warp)
    float m_new[2], corr[2];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      float mx = m_run[hs];
#pragma unroll
      for (int v = 0; v < kWarps; ++v) mx = fmaxf(mx, s_bmax[v][2 * c + hs]);
      m_new[hs] = mx;
      corr[hs] = (mx == -INFINITY) ? 1.f : expf(m_run[hs] - mx);
    }
    // weights of this warp's tokens
    float p[2][2], w[2][2];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      p[0][hs] = x[0][hs] == -INFINITY ? 0.f : expf(x[0][hs] - m_new[hs]);
      p[1][hs] = x[1][hs] == -INFINITY ? 0.f : expf(x[1][hs] - m_new[hs]);
      w[0][hs] = p[0][hs] * vn1;
      w[1][hs] = p[1][hs] * vn2;
    }
    float ps[2], wsm[2];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      float a = p[0][hs] + p[1][hs], b = w[0][hs] + w[1][hs];
      a += __shfl_xor_sync(0xffffffffu, a, 4);
      a += __shfl_xor_sync(0xffffffffu, a, 8);
      a += __shfl_xor_sync(0xffffffffu, a, 16);
      b += __shfl_xor_sync(0xffffffffu, b, 4);
      b += __shfl_xor_sync(0xffffffffu, b, 8);
      b += __shfl_xor_sync(0xffffffffu, b, 16);
      ps[hs] = a;
      wsm[hs] = b;
    }
    if (g == 0) {
      s_psum[warp][2 * c] = ps[0];
      s_psum[warp][2 * c + 1] = ps[1];
      s_wsum[warp][2 * c] = wsm[0];
      s_wsum[warp][2 * c + 1] = wsm[1];
    }
    // B operand of the value MMA: P'[token][col] with feature value 2.0 -> 0.5 w
    // rows g and g+8, columns 2c, 2c+1.  HL: columns = (head c hi, head c lo).
    // Otherwise columns = heads 2c, 2c+1 in two n-tiles (hi parts, lo parts).
    if (HL) {
      const float a = 0.5f * w[0][0], b = 0.5f * w[1][0];
      const float ah = hhi(a), bh = hhi(b);
      const uint32_t c1 = h2pack(ah, a - ah), c2 = h2pack(bh, b - bh);
      s_pb[warp][lane] = make_uint4(movtrans(c1), movtrans(c2), 0u, 0u);
    } else {
      const float a0 = 0.5f * w[0][0], a1 = 0.5f * w[0][1];
      const float b0 = 0.5f * w[1][0], b1 = 0.5f * w[1][1];
      const float a0h = hhi(a0), a1h = hhi(a1), b0h = hhi(b0), b1h = hhi(b1);
      s_pb[warp][lane] = make_uint4(movtrans(h2pack(a0h, a1h)), movtrans(h2pack(b0h, b1h)),
                                    movtrans(h2pack(a0 - a0h, a1 - a1h)),
                                    movtrans(h2pack(b0 - b0h, b1 - b1h)));
    }
    __syncthreads();

    // ================= consumer: value accumulate for coordinates [32 warp, 32 warp + 32)
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      float ls = 0.f, wss = 0.f;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) {
        ls += s_psum[v][2 * c + hs];
        wss += s_wsum[v][2 * c + hs];
      }
      l_run[hs] = l_run[hs] * corr[hs] + ls;
      w_run[hs] = w_run[hs] * corr[hs] + wss;
      m_run[hs] = m_new[hs];
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
      acc[i][0] *= corr[0];
      acc[i][1] *= HL ? corr[0] : corr[1];
      acc[i][2] *= corr[0];
      acc[i][3] *= HL ? corr[0] : corr[1];
      if (!HL) {
        accl[HL ? 0 : i][0] *= corr[0];
        accl[HL ? 0 : i][1] *= corr[1];
        accl[HL ? 0 : i][2] *= corr[0];
        accl[HL ? 0 : i][3] *= corr[1];
      }
    }
#pragma unroll
    for (int vb2 = 0; vb2 < 2; ++vb2) {
      const int64_t tb = sb + 32 * vb2;
      if (tb >= t_end) break;
      // plane words of this thread's coordinates j = 32 warp + {g, g+8, 16+g, 24+g}
      const uint32_t* vw = P.vcodes + (vblk0 + tb / 32) * (int64_t)(KV * DP);
      uint32_t pw[4][KV];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = 32 * warp + g + 8 * jj;
#pragma unroll
        for (int p = 0; p < KV; ++p) pw[jj][p] = vw[p * DP + j];
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint4 bf = s_pb[2 * vb2 + hh][lane];
        const int q0 = 8 * hh + c, q1 = 8 * hh + 4 + c;
#pragma unroll
        for (int f = 0; f < FV; ++f) {
#pragma unroll
          for (int jh = 0; jh < 2; ++jh) {
            // m-tile (f, jh): rows g -> coordinate jh*16 + g, g+8 -> jh*16 + g + 8
            const uint32_t Wa = feature_word<KV>(pw[2 * jh], f);
            const uint32_t Wb = feature_word<KV>(pw[2 * jh + 1], f);
            const uint32_t a0 = feat2(Wa, q0), a1 = feat2(Wb, q0), a2 = feat2(Wa, q1), a3 = feat2(Wb, q1);
            mma16816(acc[2 * f + jh], a0, a1, a2, a3, bf.x, bf.y);
            if (!HL) mma16816(accl[HL ? 0 : 2 * f + jh], a0, a1, a2, a3, bf.z, bf.w);
          }
        }
      }
    }
  }

  // ---- partials: o_rot_j = sum_S 2 alpha_S acc_S,j - (sum alpha) W
  float* part = P.part;
  const int d_pad = DP;
#pragma unroll
  for (int hs = 0; hs < 2; ++hs) {
    const int h = HL ? c : 2 * c + hs;
    if (h >= G || (HL && hs == 1)) continue;
#pragma unroll
    for (int jh = 0; jh < 2; ++jh) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int j = 32 * warp + 16 * jh + g + 8 * rr;
        float o = -P.valpha_sum * w_run[hs];
#pragma unroll
        for (int f = 0; f < FV; ++f) {
          const float* a4 = acc[2 * f + jh];
          const float v = HL ? (a4[2 * rr] + a4[2 * rr + 1])
                             : a4[2 * rr + hs] + accl[HL ? 0 : 2 * f + jh][2 * rr + hs];
          o = fmaf(2.f * P.valpha[f], v, o);
        }
        float* pp = part + (((int64_t)grp * P.n_chunks + chunk) * G + h) * (int64_t)(d_pad + 2);
        pp[2 + j] = o;
        if (warp == 0 && jh == 0 && rr == 0 && g == 0) {
          pp[0] = m_run[hs];
          pp[1] = l_run[hs];
        }
      }
    }
  }
}

template <int KK, int KV>
cudaError_t launch_kv(const Params& p, bool hl, dim3 grid, cudaStream_t st) {
  if (hl)
    attn_chunk_kernel<KK, KV, true><<<grid, kThreads, 0, st>>>(p);
  else
    attn_chunk_kernel<KK, KV, false><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

template <int KK>
cudaError_t launch_k(const Params& p, int kv, bool hl, dim3 grid, cudaStream_t st) {
  switch (kv) {
    case 1: return launch_kv<KK, 1>(p, hl, grid, st);
    case 2: return launch_kv<KK, 2>(p, hl, grid, st);
    case 3: return launch_kv<KK, 3>(p, hl, grid, st);
    case 4: return launch_kv<KK, 4>(p, hl, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch(const Params& p, int kk, int kv, dim3 grid, cudaStream_t st) {
  const bool hl = p.G <= 4;
  switch (kk) {
    case 1: return launch_k<1>(p, kv, hl, grid, st);
    case 2: return launch_k<2>(p, kv, hl, grid, st);
    case 3: return launch_k<3>(p, kv, hl, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn2
}  // namespace tq
