// Decode attention over a compressed KV cache with 8-bit integer tensor-core
// MMAs (turboquant-pytorch Pattern 1: scores from compressed keys, softmax,
// weighted sum of the Q_MSE-reconstructed values; TurboQuant blog notes,
// Q_prod estimator; explainer §8).
//
// Exact bit features, as in the fp16 kernel (tq_attn2.cu): a symmetric
// codebook is an odd function of the index bits, C[idx] = sum over odd subsets
// S of alpha_S (2 b_S - 1), b_S the XOR of the bits in S, so every
// contraction is against 0/1 bit matrices:
//   <q', C[idx]>         = sum_S alpha_S (2 <q', b_S> - sum q'),
//   <u, 2 sigma - 1>     = 2 <u, sigma> - sum u,
//   sum_t w_t C[idx_t]_j = sum_S alpha_S (2 sum_t w_t b_S,tj - sum_t w_t).
//
// Operands.  A bit matrix enters the MMA as unsigned bytes {0, 128}: four bits
// of a code word that are 8 apart land on the four byte sign positions with
// one multiply by a power of two and one AND (the K order is permuted the same
// way on both operands).  The other operand is a fixed-point integer split
// into exact bytes.  Queries q' and u: 24 bits with a per-head scale
// max|.| / (127 * 2^16), signed bytes hi, mid, lo; hi and mid of heads 4 nt ..
// 4 nt + 3 fill N-tile nt (columns 2 h, 2 h + 1), the lo bytes of all heads
// one more tile (columns 2 h' and 2 h' + 1 hold heads h' and 4 + h', so each
// thread meets the same heads in every tile).  Softmax weights p ||v||: 16
// bits with a per-head scale (their maximum over the sub-chunk) / 65535,
// unsigned bytes hi, lo in adjacent columns (four heads per tile).  Products
// and sums are exact integers; the only rounding is the fixed point itself
// (2^-24 of the largest query entry, 2^-16 of the largest weight).
//
// Per CTA: one (layer, batch, kv-head) group and one chunk, 4 warps, in
// sub-chunks of up to 512 tokens:
//   A. scores: warp w takes 16-token m-tiles w, w + 4, ... (rows = tokens,
//      K = the 32 coordinates of one plane word, N = heads x {hi, lo}); the
//      scores go to shared memory, with the sub-chunk maximum per head;
//   B. weights p = exp(s - m) ||v|| (m the running maximum) as 16-bit fixed
//      point, stored as bytes in B-fragment order;
//   C. values: warp w accumulates its 32 value coordinates (rows = coordinate
//      features, K = the 32 tokens of one BLOCK32 word, N = heads x {hi, lo}).
// The integer accumulators are folded into fp32 running (m, l, o) after each
// sub-chunk; the partial (m, l, o_rot) of the chunk goes to the workspace for
// the combine kernel.
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_attn2.h"
#include "tq_attn3.h"
#include "tq_device.cuh"

namespace tq {
namespace attn3 {

using attn2::Params;

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int DP = 128;            // rotated dimension
constexpr int WPP = DP / 32;       // words per code plane
constexpr int M = 128;             // QJL rows
constexpr int SW = M / 32;         // sign words per token
constexpr int SC = 512;            // tokens per sub-chunk
constexpr float kQMax = 8323072.0f;  // 127 * 2^16: the hi byte stays in [-127, 127]

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_u8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bytes {0, 128} from bits s0 + 8 i (i = 0..3) of w, mul = 2^(7 - s0): the
// multiply moves them to the byte sign positions.
__device__ __forceinline__ uint32_t bits_to_bytes(uint32_t w, uint32_t mul) {
  return (w * mul) & 0x80808080u;
}

template <int K>
struct NF {  // odd-subset features of a k-bit code: 2^(k-1)
  static constexpr int v = 1 << (K - 1);
};

// Feature word S from the k plane words p[0..k): odd subsets in the order
// {0},{1},...,{k-1}, then the triples.
template <int K>
__device__ __forceinline__ uint32_t feature_word(const uint32_t* p, int f) {
  if (f < K) return p[f];
  const int t = f - K;
  if (K == 3) return p[0] ^ p[1] ^ p[2];
  const int skip = 3 - t;  // the element left out of the 4-set
  uint32_t x = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q != skip) x ^= p[q];
  return x;
}

// Byte `piece` (0: hi, 1: mid, 2: lo) of the 24-bit fixed point
// v = round(x * inv), |v| <= 127 * 2^16, written as v = 2^16 hi + 2^8 mid + lo
// with balanced digits: lo = ((v + 128) mod 256) - 128, then the same for
// (v - lo) / 256; every digit lies in [-128, 127].
__device__ __forceinline__ uint32_t fixed_byte(float x, float inv, int piece) {
  const int v = __float2int_rn(x * inv);
  const int lo = ((v + 128) & 0xFF) - 128;
  const int v1 = (v - lo) >> 8;  // exact
  const int mid = ((v1 + 128) & 0xFF) - 128;
  const int hi = (v1 - mid) >> 8;
  return (uint32_t)((piece == 0 ? hi : piece == 1 ? mid : lo) & 0xFF);
}

template <int KK, int KV, int NT>
__global__ void __launch_bounds__(kThreads) attn_kernel(Params P) {
  constexpr int FK = NF<KK>::v;  // key code features
  constexpr int FV = NF<KV>::v;  // value code features
  constexpr int KW = KK * WPP;   // key code words per token
  constexpr int HN = 4 * NT;     // head slots

  __shared__ float s_score[SC][HN];  // scores, then weights p ||v||
  __shared__ __align__(16) uint32_t s_wb[SC / 32][NT][8][4][2];  // weight bytes, B-fragment order
  __shared__ float s_qf[2][HN][DP];  // q' and u (M = DP) of the heads
  __shared__ float s_red[3][kWarps][HN];
  __shared__ float s_head[HN][8];  // per head: Qq, Qu, sum q_int, sum u_int, m, l, 1/Qq, 1/Qu

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int G = P.G;
  const int grp = blockIdx.y, chunk = blockIdx.x;
  // K slots 4 tig + i <-> bits 2 tig + 8 i, 16 + 4 tig + i <-> bits 2 tig + 1 + 8 i
  const uint32_t mul0 = 1u << (7 - 2 * tig), mul1 = 1u << (6 - 2 * tig);

  // ---- query side: fixed-point scales and the score B fragments
  for (int e = tid; e < 2 * HN * DP; e += kThreads) {
    const int which = e / (HN * DP), h = (e / DP) % HN, j = e % DP;
    float x = 0.f;
    if (h < G) x = which == 0 ? P.qrot[((int64_t)grp * G + h) * DP + j] : P.u[((int64_t)grp * G + h) * M + j];
    s_qf[which][h][j] = x;
  }
  for (int e = tid; e < (SC / 32) * NT * 8 * 4 * 2; e += kThreads) (&s_wb[0][0][0][0][0])[e] = 0u;
  __syncthreads();
  for (int hw = warp; hw < 2 * HN; hw += kWarps) {  // (which, head) per warp
    const int which = hw / HN, h = hw % HN;
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fabsf(s_qf[which][h][lane + 32 * i]));
    mx = warp_max(mx);
    const float inv = mx > 0.f ? kQMax / mx : 0.f;
    int sum = 0;  // |sum| <= 128 * 127 * 2^16 < 2^31
#pragma unroll
    for (int i = 0; i < 4; ++i) sum += __float2int_rn(s_qf[which][h][lane + 32 * i] * inv);
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0) {
      s_head[h][which] = mx / kQMax;      // Qq or Qu
      s_head[h][2 + which] = (float)sum;  // sum of q_int or u_int
      s_head[h][6 + which] = inv;
    }
  }
  if (tid < HN) {
    s_head[tid][4] = -INFINITY;  // running max
    s_head[tid][5] = 0.f;        // running sum of p
  }
  __syncthreads();
  // B fragments, column g of tile nt < NT: head 4 nt + g / 2, piece hi (g
  // even) or mid; of tile NT: head g / 2 (g even) or 4 + g / 2, piece lo.  For
  // plane word cw, b0 bytes = coordinates 32 cw + 2 tig + 8 i and b1 =
  // 32 cw + 2 tig + 1 + 8 i.
  uint32_t bq[NT + 1][2][WPP][2];
#pragma unroll
  for (int nt = 0; nt <= NT; ++nt) {
    const int hc = nt < NT ? 4 * nt + (g >> 1) : (g & 1) * 4 + (g >> 1);
    const bool hv = hc < HN;  // lo tile with one head tile: columns of heads 4..7 are zero
    const int h = hv ? hc : 0;
    const int piece = nt < NT ? (g & 1) : 2;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const float inv = s_head[h][6 + which];
#pragma unroll
      for (int cw = 0; cw < WPP; ++cw) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          uint32_t w = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            w |= fixed_byte(s_qf[which][h][32 * cw + 2 * tig + r + 8 * i], inv, piece) << (8 * i);
          bq[nt][which][cw][r] = hv ? w : 0u;
        }
      }
    }
  }
  // per thread-column heads (4 nt + tig): score constants
  float cA1[NT], cC1[NT], cA2[NT], cC2[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = 4 * nt + tig;
    const float Qq = s_head[h][0], Qu = s_head[h][1];
    cA1[nt] = Qq * (1.0f / 64.0f);                // <q', b> = Qq v / 128, times 2
    cC1[nt] = -Qq * P.kalpha_sum * s_head[h][2];  // - sum_S alpha_S sum q'
    cA2[nt] = P.kappa * Qu * (1.0f / 64.0f);
    cC2[nt] = -P.kappa * Qu * s_head[h][3];
  }

  const int64_t t_begin = (int64_t)chunk * P.chunk;
  const int64_t t_end = min64(P.seq, t_begin + P.chunk);
  const int64_t krow0 = (int64_t)grp * P.cap;
  const int64_t vblk0 = (int64_t)grp * (P.cap / 32);
  const float scale = P.scale;
  float o_run[NT][2][2];  // [nt][jh][row]: coordinate 32 warp + 16 jh + g + 8 row, head 4 nt + tig
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int jh = 0; jh < 2; ++jh) o_run[nt][jh][0] = o_run[nt][jh][1] = 0.f;

  for (int64_t s0 = t_begin; s0 < t_end; s0 += SC) {
    const int scn = (int)min64(SC, t_end - s0);  // tokens of this sub-chunk
    // ================= A. scores
    float mloc[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mloc[nt] = -INFINITY;
    for (int mt = warp; 16 * mt < scn; mt += kWarps) {
      const int l1 = 16 * mt + g, l2 = l1 + 8;
      const bool ok1 = l1 < scn, ok2 = l2 < scn;
      const int64_t R1 = krow0 + s0 + (ok1 ? l1 : scn - 1), R2 = krow0 + s0 + (ok2 ? l2 : scn - 1);
      uint32_t k1[KW + SW], k2[KW + SW];
#pragma unroll
      for (int i = 0; i < KW; i += 4) {
        const uint4 a = *reinterpret_cast<const uint4*>(P.kcodes + R1 * KW + i);
        const uint4 b = *reinterpret_cast<const uint4*>(P.kcodes + R2 * KW + i);
        k1[i] = a.x; k1[i + 1] = a.y; k1[i + 2] = a.z; k1[i + 3] = a.w;
        k2[i] = b.x; k2[i + 1] = b.y; k2[i + 2] = b.z; k2[i + 3] = b.w;
      }
      {
        const uint4 a = *reinterpret_cast<const uint4*>(P.ksigns + R1 * SW);
        const uint4 b = *reinterpret_cast<const uint4*>(P.ksigns + R2 * SW);
        k1[KW] = a.x; k1[KW + 1] = a.y; k1[KW + 2] = a.z; k1[KW + 3] = a.w;
        k2[KW] = b.x; k2[KW + 1] = b.y; k2[KW + 2] = b.z; k2[KW + 3] = b.w;
      }
      const float n1 = P.knorms[R1], n2 = P.knorms[R2];
      const float r1 = P.krnorms[R1], r2 = P.krnorms[R2];
      int acc[FK + 1][NT + 1][4];
#pragma unroll
      for (int f = 0; f <= FK; ++f)
#pragma unroll
        for (int nt = 0; nt <= NT; ++nt) acc[f][nt][0] = acc[f][nt][1] = acc[f][nt][2] = acc[f][nt][3] = 0;
#pragma unroll
      for (int cw = 0; cw < WPP; ++cw) {
        uint32_t p1[KK], p2[KK];
#pragma unroll
        for (int p = 0; p < KK; ++p) {
          p1[p] = k1[p * WPP + cw];
          p2[p] = k2[p * WPP + cw];
        }
#pragma unroll
        for (int f = 0; f <= FK; ++f) {
          // features of the key code, then the QJL sign plane
          const uint32_t W1 = f < FK ? feature_word<KK>(p1, f) : k1[KW + cw];
          const uint32_t W2 = f < FK ? feature_word<KK>(p2, f) : k2[KW + cw];
          const uint32_t a0 = bits_to_bytes(W1, mul0), a1 = bits_to_bytes(W2, mul0);
          const uint32_t a2 = bits_to_bytes(W1, mul1), a3 = bits_to_bytes(W2, mul1);
          const int which = f < FK ? 0 : 1;
#pragma unroll
          for (int nt = 0; nt <= NT; ++nt)
            mma_u8s8(acc[f][nt], a0, a1, a2, a3, bq[nt][which][cw][0], bq[nt][which][cw][1]);
        }
      }
      // s = scale n (Qq (sum_S alpha_S v_S / 64 - sum alpha sum q_int)
      //              + kappa rho Qu (v_sign / 64 - sum u_int)),
      // v = 2^16 hi + 2^8 mid + lo (hi, mid: tile nt; lo: tile NT, column nt)
      auto comb = [&](const int (&t)[NT + 1][4], int nt, int row) {
        return fmaf(65536.f, (float)t[nt][2 * row], fmaf(256.f, (float)t[nt][2 * row + 1], (float)t[NT][2 * row + nt]));
      };
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int h = 4 * nt + tig;
        float m1 = 0.f, m2 = 0.f;
#pragma unroll
        for (int f = 0; f < FK; ++f) {
          m1 = fmaf(P.kalpha[f], comb(acc[f], nt, 0), m1);
          m2 = fmaf(P.kalpha[f], comb(acc[f], nt, 1), m2);
        }
        const float q1 = comb(acc[FK], nt, 0);
        const float q2 = comb(acc[FK], nt, 1);
        const float x1 = scale * n1 * (fmaf(cA1[nt], m1, cC1[nt]) + r1 * fmaf(cA2[nt], q1, cC2[nt]));
        const float x2 = scale * n2 * (fmaf(cA1[nt], m2, cC1[nt]) + r2 * fmaf(cA2[nt], q2, cC2[nt]));
        if (h < G) {
          if (ok1) s_score[l1][h] = x1;
          if (ok2) s_score[l2][h] = x2;
          mloc[nt] = fmaxf(mloc[nt], fmaxf(ok1 ? x1 : -INFINITY, ok2 ? x2 : -INFINITY));
        }
      }
    }
    // sub-chunk maximum per head (over g: lanes xor 4, 8, 16; then warps)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float v = mloc[nt];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      if (g == 0) s_red[0][warp][4 * nt + tig] = v;
    }
    __syncthreads();
    // ================= B. weights
    // thread tid: tokens tid, tid + 128, ... of the sub-chunk, every head
    float mnew[HN], lpart[HN], wmax[HN];
#pragma unroll
    for (int h = 0; h < HN; ++h) {
      float mx = s_head[h][4];
#pragma unroll
      for (int v = 0; v < kWarps; ++v) mx = fmaxf(mx, s_red[0][v][h]);
      mnew[h] = mx;
      lpart[h] = 0.f;
      wmax[h] = 0.f;
    }
    for (int t = tid; t < scn; t += kThreads) {
      const float vn = P.vnorms[krow0 + s0 + t];
#pragma unroll
      for (int h = 0; h < HN; ++h) {
        if (h < G) {
          const float s = s_score[t][h];
          const float p = s == -INFINITY ? 0.f : expf(s - mnew[h]);
          const float w = p * vn;
          s_score[t][h] = w;
          lpart[h] += p;
          wmax[h] = fmaxf(wmax[h], w);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < HN; ++h) {
      float a = warp_sum(lpart[h]), b = warp_max(wmax[h]);
      if (lane == 0) {
        s_red[1][warp][h] = a;
        s_red[2][warp][h] = b;
      }
    }
    __syncthreads();
    float winv[HN];
#pragma unroll
    for (int h = 0; h < HN; ++h) {
      float mx = 0.f;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) mx = fmaxf(mx, s_red[2][v][h]);
      winv[h] = mx > 0.f ? 65535.0f / mx : 0.f;
    }
    int wsum[HN];
#pragma unroll
    for (int h = 0; h < HN; ++h) wsum[h] = 0;
    // weight bytes: token tau of a 32-token block sits in K slot 4 tg + i
    // (register r) with tau = 2 tg + r + 8 i
    const int scn32 = (scn + 31) & ~31;
    for (int t = tid; t < scn32; t += kThreads) {
      const int blk = t >> 5, tau = t & 31;
      const int tg = (tau & 7) >> 1, r = tau & 1, i = tau >> 3;
#pragma unroll
      for (int h = 0; h < HN; ++h) {
        if (h < G) {
          const int wi = t < scn ? __float2int_rn(s_score[t][h] * winv[h]) : 0;
          wsum[h] += wi;
          unsigned char* hb = reinterpret_cast<unsigned char*>(&s_wb[blk][h >> 2][2 * (h & 3)][tg][r]);
          unsigned char* lb = reinterpret_cast<unsigned char*>(&s_wb[blk][h >> 2][2 * (h & 3) + 1][tg][r]);
          hb[i] = (unsigned char)(wi >> 8);
          lb[i] = (unsigned char)(wi & 0xFF);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < HN; ++h) {
      const int a = __reduce_add_sync(0xffffffffu, wsum[h]);
      if (lane == 0) s_red[0][warp][h] = __int_as_float(a);
    }
    __syncthreads();
    // running softmax state of the thread's column heads
    float corr[NT], wscale[NT], wtot[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = 4 * nt + tig;
      float mn = 0.f, wi = 0.f;
#pragma unroll
      for (int hh = 4 * nt; hh < 4 * nt + 4; ++hh) {  // register select of head h
        mn = hh == h ? mnew[hh] : mn;
        wi = hh == h ? winv[hh] : wi;
      }
      const float mold = s_head[h][4];
      corr[nt] = mold == -INFINITY ? 0.f : expf(mold - mn);
      wscale[nt] = wi > 0.f ? 1.0f / wi : 0.f;
      int ws = 0;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) ws += __float_as_int(s_red[0][v][h]);
      wtot[nt] = (float)ws;
    }
    // ================= C. values: coordinates 32 warp + 16 jh + g + 8 row
    int accv[FV][2][NT][4];
#pragma unroll
    for (int f = 0; f < FV; ++f)
#pragma unroll
      for (int jh = 0; jh < 2; ++jh)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) accv[f][jh][nt][0] = accv[f][jh][nt][1] = accv[f][jh][nt][2] = accv[f][jh][nt][3] = 0;
    for (int blk = 0; 32 * blk < scn; ++blk) {
      const uint32_t* vw = P.vcodes + (vblk0 + s0 / 32 + blk) * (int64_t)(KV * DP);
      uint32_t pw[2][2][KV];
#pragma unroll
      for (int jh = 0; jh < 2; ++jh)
#pragma unroll
        for (int rw = 0; rw < 2; ++rw) {
          const int j = 32 * warp + 16 * jh + g + 8 * rw;
#pragma unroll
          for (int p = 0; p < KV; ++p) pw[jh][rw][p] = vw[p * DP + j];
        }
      uint2 bw[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) bw[nt] = *reinterpret_cast<const uint2*>(&s_wb[blk][nt][g][tig][0]);
#pragma unroll
      for (int f = 0; f < FV; ++f) {
#pragma unroll
        for (int jh = 0; jh < 2; ++jh) {
          const uint32_t Wa = feature_word<KV>(pw[jh][0], f), Wb = feature_word<KV>(pw[jh][1], f);
          const uint32_t a0 = bits_to_bytes(Wa, mul0), a1 = bits_to_bytes(Wb, mul0);
          const uint32_t a2 = bits_to_bytes(Wa, mul1), a3 = bits_to_bytes(Wb, mul1);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_u8u8(accv[f][jh][nt], a0, a1, a2, a3, bw[nt].x, bw[nt].y);
        }
      }
    }
    // fold: o += w_scale (sum_S alpha_S v_S / 64 - sum alpha W), v = 256 hi + lo
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int jh = 0; jh < 2; ++jh) {
#pragma unroll
        for (int rw = 0; rw < 2; ++rw) {
          float s = 0.f;
#pragma unroll
          for (int f = 0; f < FV; ++f)
            s = fmaf(P.valpha[f], fmaf(256.f, (float)accv[f][jh][nt][2 * rw], (float)accv[f][jh][nt][2 * rw + 1]), s);
          const float o_sub = wscale[nt] * fmaf(s, 1.0f / 64.0f, -P.valpha_sum * wtot[nt]);
          o_run[nt][jh][rw] = fmaf(o_run[nt][jh][rw], corr[nt], o_sub);
        }
      }
    }
    __syncthreads();  // every thread has read s_head / s_red / s_wb of this sub-chunk
    if (tid < HN && tid < G) {
      float ls = 0.f, mn = 0.f;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) ls += s_red[1][v][tid];
#pragma unroll
      for (int hh = 0; hh < HN; ++hh) mn = hh == tid ? mnew[hh] : mn;
      const float mold = s_head[tid][4];
      const float c = mold == -INFINITY ? 0.f : expf(mold - mn);
      s_head[tid][5] = s_head[tid][5] * c + ls;
      s_head[tid][4] = mn;
    }
    __syncthreads();
  }

  // ---- partial (m, l, o_rot) of this chunk
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = 4 * nt + tig;
    if (h >= G) continue;
    float* pp = P.part + (((int64_t)grp * P.n_chunks + chunk) * G + h) * (int64_t)(DP + 2);
#pragma unroll
    for (int jh = 0; jh < 2; ++jh)
#pragma unroll
      for (int rw = 0; rw < 2; ++rw) pp[2 + 32 * warp + 16 * jh + g + 8 * rw] = o_run[nt][jh][rw];
    if (warp == 0 && g == 0) {
      pp[0] = s_head[h][4];
      pp[1] = s_head[h][5];
    }
  }
}

template <int KK, int KV>
cudaError_t launch_kv(const Params& p, dim3 grid, cudaStream_t st) {
  if (p.G <= 4)
    attn_kernel<KK, KV, 1><<<grid, kThreads, 0, st>>>(p);
  else
    attn_kernel<KK, KV, 2><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

template <int KK>
cudaError_t launch_k(const Params& p, int kv, dim3 grid, cudaStream_t st) {
  switch (kv) {
    case 1: return launch_kv<KK, 1>(p, grid, st);
    case 2: return launch_kv<KK, 2>(p, grid, st);
    case 3: return launch_kv<KK, 3>(p, grid, st);
    case 4: return launch_kv<KK, 4>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch(const Params& p, int kk, int kv, dim3 grid, cudaStream_t st) {
  if (p.G < 1 || p.G > 8) return cudaErrorInvalidValue;
  switch (kk) {
    case 1: return launch_k<1>(p, kv, grid, st);
    case 2: return launch_k<2>(p, kv, grid, st);
    case 3: return launch_k<3>(p, kv, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn3
}  // namespace tq
