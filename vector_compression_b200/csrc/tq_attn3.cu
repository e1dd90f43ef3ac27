// Decode attention over a compressed KV cache with 8-bit integer tensor-core
// MMAs (turboquant-pytorch Pattern 1: scores from compressed keys, softmax,
// weighted sum of the Q_MSE-reconstructed values; TurboQuant blog notes,
// Q_prod estimator; explainer §8).
//
// Exact bit features: a symmetric
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
// Per CTA: one (layer, batch, kv-head) group and one chunk, d_pad / 32 warps
// (4 at d_pad 128, 8 at 256), in sub-chunks of up to 384 (d_pad 128) or 192
// (d_pad 256) tokens whose keys, value blocks and norms are
// staged in shared memory by bulk asynchronous copies (the next sub-chunk's
// keys load while this one's weights and values are formed, its values while
// the next scores are):
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

#include "tq_attn_params.h"
#include "tq_attn3.h"
#include "tq_device.cuh"
#include "tq_wait.cuh"

namespace tq {
namespace attn3 {

using attn::Params;

// The geometry (warps, words per plane, sub-chunk length) follows d_pad:
// see Layout.
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
  uint32_t r;  // an integer multiply (FMA pipe), not a shift (ALU pipe)
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(mul));
  return r & 0x80808080u;
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

// Shared-memory layout of one CTA (bytes): the staged sub-chunk (key codes,
// sign words, key norms, residual norms | value blocks, value norms), scores
// (which first hold the query rows during setup) and weight bytes.
template <int KK, int KV, int NT, int MQ, int DPT>
struct Layout {
  // d_pad 256: one warp per 32 value coordinates (eight warps) and 192-token
  // sub-chunks; the query fragments live in shared memory
  static constexpr int DP = DPT, WPP = DPT / 32, SC = DPT == 128 ? 384 : 192;
  static constexpr int KW = KK * WPP, HN = 4 * NT, SW = MQ / 32;
  static constexpr int SROWS = SC > 2 * DP ? SC : 2 * DP;  // score rows (query rows during setup)
  static constexpr uint32_t kc = 0;
  static constexpr uint32_t ks = kc + SC * KW * 4;
  static constexpr uint32_t kn = ks + SC * SW * 4;
  static constexpr uint32_t kr = kn + SC * 4;
  static constexpr uint32_t vc = kr + SC * 4;
  static constexpr uint32_t vn = vc + (SC / 32) * KV * DP * 4;
  static constexpr uint32_t score = vn + SC * 4;
  static constexpr uint32_t wb = score + SROWS * HN * 4;
  static constexpr uint32_t bq = wb + (SC / 32) * NT * 8 * 4 * 2 * 4;
  static constexpr uint32_t bytes = bq + (DPT == 128 ? 0 : (NT + 1) * 2 * WPP * 32 * 8);
  // the query rows (setup only) share the score buffer
  static constexpr uint32_t qf = score;
  static_assert(SROWS * HN >= 2 * HN * DP, "query rows fit in the score buffer");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// global to shared memory, completing on the mbarrier.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait for the phase with the given parity: false, and the device
// error word set (when err is not null), if it does not complete within the
// wait budget.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* err) {
  return bounded_wait<true>(bar, parity, err);
}

template <int KK, int KV, int NT, int MQ, int DPT>
__global__ void __launch_bounds__(DPT) attn_kernel(Params P) {
  using LY = Layout<KK, KV, NT, MQ, DPT>;
  // geometry of this d_pad (shadows the d_pad = 128 constants above)
  constexpr int DP = LY::DP, WPP = LY::WPP, SC = LY::SC;
  constexpr int kWarps = DPT / 32, kThreads = DPT;
  constexpr int SW = MQ / 32;    // QJL sign words per token (m / 32)
  constexpr int FK = NF<KK>::v;  // key code features
  constexpr int FV = NF<KV>::v;  // value code features
  constexpr int KW = KK * WPP;   // key code words per token
  constexpr int HN = 4 * NT;     // head slots
  constexpr float kLog2e = 1.4426950408889634f;

  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* s_kc = reinterpret_cast<uint32_t*>(smem + LY::kc);   // [SC][KW]
  uint32_t* s_ks = reinterpret_cast<uint32_t*>(smem + LY::ks);   // [SC][SW]
  float* s_kn = reinterpret_cast<float*>(smem + LY::kn);         // [SC]
  float* s_kr = reinterpret_cast<float*>(smem + LY::kr);         // [SC]
  uint32_t* s_vc = reinterpret_cast<uint32_t*>(smem + LY::vc);   // [SC/32][KV*DP]
  float* s_vn = reinterpret_cast<float*>(smem + LY::vn);         // [SC]
  float (*s_score)[HN] = reinterpret_cast<float (*)[HN]>(smem + LY::score);  // log2-domain scores, then weights
  static_assert(LY::score % 16 == 0, "vector access to the score rows");
  uint32_t (*s_wb)[NT][8][4][2] = reinterpret_cast<uint32_t (*)[NT][8][4][2]>(smem + LY::wb);
  float (*s_qf)[HN][DP] = reinterpret_cast<float (*)[HN][DP]>(smem + LY::qf);
  uint2 (*s_bq)[2][WPP][32] = reinterpret_cast<uint2 (*)[2][WPP][32]>(smem + LY::bq);  // d_pad 256
  __shared__ __align__(8) uint64_t bar_k, bar_v;
  __shared__ float s_red[3][kWarps][HN];
  __shared__ float s_head[HN][8];  // per head: Qq, Qu, sum q_int, sum u_int, m, l, 1/Qq, 1/Qu

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int G = P.G;
  const int grp = blockIdx.y, chunk = blockIdx.x;
  const int64_t t_begin = (int64_t)chunk * P.chunk;
  const int64_t t_end = min64(P.seq, t_begin + P.chunk);
  const int64_t krow0 = (int64_t)grp * P.cap;
  const int64_t vblk0 = (int64_t)grp * (P.cap / 32);
  // K slots 4 tig + i <-> bits 2 tig + 8 i, 16 + 4 tig + i <-> bits 2 tig + 1 + 8 i
  const uint32_t mul0 = 1u << (7 - 2 * tig), mul1 = 1u << (6 - 2 * tig);

  // ---- staging of sub-chunks (one thread issues the bulk copies)
  const uint32_t bk = smem_u32(&bar_k), bv = smem_u32(&bar_v);
  // keys of the sub-chunk at s: codes, signs, norms, residual norms of
  // round_up(n, 4) tokens (inside the cache: cap >= round_up(seq, 32))
  auto issue_keys = [&](int64_t s) {
    const uint32_t n4 = (uint32_t)((min64(SC, t_end - s) + 3) & ~3);
    // fp16 residual norms: 8-token granules keep the copy a multiple of 16 bytes
    const uint32_t kr_bytes = P.kr16 ? ((n4 + 7) & ~7u) * 2 : n4 * 4;
    mbar_expect(bk, n4 * (KW * 4 + SW * 4 + 4) + kr_bytes);
    bulk_g2s(s_kc, P.kcodes + (krow0 + s) * KW, n4 * KW * 4, bk);
    bulk_g2s(s_ks, P.ksigns + (krow0 + s) * SW, n4 * SW * 4, bk);
    bulk_g2s(s_kn, P.knorms + krow0 + s, n4 * 4, bk);
    bulk_g2s(s_kr, reinterpret_cast<const char*>(P.krnorms) + (krow0 + s) * (P.kr16 ? 2 : 4), kr_bytes, bk);
  };
  // values of the sub-chunk at s: its 32-token blocks and the value norms
  auto issue_values = [&](int64_t s) {
    const int64_t n = min64(SC, t_end - s);
    const uint32_t nb = (uint32_t)((n + 31) / 32), n4 = (uint32_t)((n + 3) & ~3);
    mbar_expect(bv, nb * KV * DP * 4 + n4 * 4);
    bulk_g2s(s_vc, P.vcodes + (vblk0 + s / 32) * (int64_t)(KV * DP), nb * KV * DP * 4, bv);
    bulk_g2s(s_vn, P.vnorms + krow0 + s, n4 * 4, bv);
  };
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bk));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bv));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    issue_keys(t_begin);
    issue_values(t_begin);
  }

  // ---- query side: fixed-point scales and the score B fragments
  for (int e = tid; e < 2 * HN * DP; e += kThreads) {
    const int which = e / (HN * DP), h = (e / DP) % HN, j = e % DP;
    float x = 0.f;
    if (h < G && (which == 0 || j < MQ))
      x = which == 0 ? P.qrot[((int64_t)grp * G + h) * DP + j] : P.u[((int64_t)grp * G + h) * MQ + j];
    s_qf[which][h][j] = x;
  }
  for (int e = tid; e < (SC / 32) * NT * 8 * 4 * 2; e += kThreads) (&s_wb[0][0][0][0][0])[e] = 0u;
  __syncthreads();
  for (int hw = warp; hw < 2 * HN; hw += kWarps) {  // (which, head) per warp
    const int which = hw / HN, h = hw % HN;
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < WPP; ++i) mx = fmaxf(mx, fabsf(s_qf[which][h][lane + 32 * i]));
    mx = warp_max(mx);
    const float inv = mx > 0.f ? kQMax / mx : 0.f;
    int sum = 0;  // |sum| <= d_pad * 127 * 2^16 < 2^31 for d_pad <= 256
#pragma unroll
    for (int i = 0; i < WPP; ++i) sum += __float2int_rn(s_qf[which][h][lane + 32 * i] * inv);
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0) {
      s_head[h][which] = mx / kQMax;      // Qq or Qu
      s_head[h][2 + which] = (float)sum;  // sum of q_int or u_int
      s_head[h][6 + which] = inv;
    }
  }
  if (tid < HN) {
    s_head[tid][4] = -INFINITY;  // running max (log2 domain)
    s_head[tid][5] = 0.f;        // running sum of p
  }
  __syncthreads();
  // B fragments, column g of tile nt < NT: head 4 nt + g / 2, piece hi (g
  // even) or mid; of tile NT: head g / 2 (g even) or 4 + g / 2, piece lo.  For
  // plane word cw, b0 bytes = coordinates 32 cw + 2 tig + 8 i and b1 =
  // 32 cw + 2 tig + 1 + 8 i.
  // d_pad 128: in registers; d_pad 256: in shared memory (the same for every
  // warp; warp 0 writes them)
  uint32_t bq[DPT == 128 ? NT + 1 : 1][2][DPT == 128 ? WPP : 1][2];
  if (DPT == 128 || warp == 0) {
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
          uint32_t w2[2];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            uint32_t w = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w |= fixed_byte(s_qf[which][h][32 * cw + 2 * tig + r + 8 * i], inv, piece) << (8 * i);
            w2[r] = hv ? w : 0u;
          }
          if constexpr (DPT == 128) {
            bq[nt][which][cw][0] = w2[0];
            bq[nt][which][cw][1] = w2[1];
          } else {
            s_bq[nt][which][cw][lane] = make_uint2(w2[0], w2[1]);
          }
        }
      }
    }
  }
  auto bfrag = [&](int nt, int which, int cw) -> uint2 {
    if constexpr (DPT == 128) return make_uint2(bq[nt][which][cw][0], bq[nt][which][cw][1]);
    else return s_bq[nt][which][cw][lane];
  };
  __syncthreads();  // the query rows (in the score buffer) have been read
  // per thread-column heads (4 nt + tig): score constants, log2 domain
  float cA1[NT], cC1[NT], cA2[NT], cC2[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = 4 * nt + tig;
    const float Qq = s_head[h][0], Qu = s_head[h][1];
    const float sl = P.scale * kLog2e;
    cA1[nt] = sl * Qq * (1.0f / 64.0f);                // <q', b> = Qq v / 128, times 2
    cC1[nt] = -sl * Qq * P.kalpha_sum * s_head[h][2];  // - sum_S alpha_S sum q'
    cA2[nt] = sl * P.kappa * Qu * (1.0f / 64.0f);
    cC2[nt] = -sl * P.kappa * Qu * s_head[h][3];
  }

  float o_run[NT][2][2];  // [nt][jh][row]: coordinate 32 warp + 16 jh + g + 8 row, head 4 nt + tig
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int jh = 0; jh < 2; ++jh) o_run[nt][jh][0] = o_run[nt][jh][1] = 0.f;

  uint32_t phase = 0;
  bool ok = true;
  for (int64_t s0 = t_begin; s0 < t_end; s0 += SC, phase ^= 1u) {
    const int scn = (int)min64(SC, t_end - s0);  // tokens of this sub-chunk
    // ================= A. scores (log2 domain) from the staged keys
    bool okw = mbar_wait(bk, phase, P.err);
    float mloc[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mloc[nt] = -INFINITY;
    for (int mt = warp; okw && 16 * mt < scn; mt += kWarps) {
      const int l1 = 16 * mt + g, l2 = l1 + 8;
      const bool ok1 = l1 < scn, ok2 = l2 < scn;
      const int R1 = ok1 ? l1 : scn - 1, R2 = ok2 ? l2 : scn - 1;
      uint32_t k1[KW + SW], k2[KW + SW];
#pragma unroll
      for (int i = 0; i < KW; i += 4) {
        const uint4 a = *reinterpret_cast<const uint4*>(s_kc + R1 * KW + i);
        const uint4 b = *reinterpret_cast<const uint4*>(s_kc + R2 * KW + i);
        k1[i] = a.x; k1[i + 1] = a.y; k1[i + 2] = a.z; k1[i + 3] = a.w;
        k2[i] = b.x; k2[i + 1] = b.y; k2[i + 2] = b.z; k2[i + 3] = b.w;
      }
      if (SW % 4 == 0) {
#pragma unroll
        for (int i = 0; i < SW; i += 4) {
          const uint4 a = *reinterpret_cast<const uint4*>(s_ks + R1 * SW + i);
          const uint4 b = *reinterpret_cast<const uint4*>(s_ks + R2 * SW + i);
          k1[KW + i] = a.x; k1[KW + i + 1] = a.y; k1[KW + i + 2] = a.z; k1[KW + i + 3] = a.w;
          k2[KW + i] = b.x; k2[KW + i + 1] = b.y; k2[KW + i + 2] = b.z; k2[KW + i + 3] = b.w;
        }
      } else {
        const uint2 a = *reinterpret_cast<const uint2*>(s_ks + R1 * SW);
        const uint2 b = *reinterpret_cast<const uint2*>(s_ks + R2 * SW);
        k1[KW] = a.x; k1[KW + 1] = a.y;
        k2[KW] = b.x; k2[KW + 1] = b.y;
      }
      const float n1 = s_kn[R1], n2 = s_kn[R2];
      const float r1 = P.kr16 ? __half2float(reinterpret_cast<const __half*>(s_kr)[R1]) : s_kr[R1];
      const float r2 = P.kr16 ? __half2float(reinterpret_cast<const __half*>(s_kr)[R2]) : s_kr[R2];
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
          if (f == FK && cw >= SW) continue;  // the sign plane has m / 32 words
          // features of the key code, then the QJL sign plane
          const uint32_t W1 = f < FK ? feature_word<KK>(p1, f) : k1[KW + cw];
          const uint32_t W2 = f < FK ? feature_word<KK>(p2, f) : k2[KW + cw];
          const uint32_t a0 = bits_to_bytes(W1, mul0), a1 = bits_to_bytes(W2, mul0);
          const uint32_t a2 = bits_to_bytes(W1, mul1), a3 = bits_to_bytes(W2, mul1);
          const int which = f < FK ? 0 : 1;
#pragma unroll
          for (int nt = 0; nt <= NT; ++nt) {
            const uint2 bb = bfrag(nt, which, cw);
            mma_u8s8(acc[f][nt], a0, a1, a2, a3, bb.x, bb.y);
          }
        }
      }
      // s log2(e) = scale log2(e) n (Qq (sum_S alpha_S v_S / 64 - sum alpha sum q_int)
      //                     + kappa rho Qu (v_sign / 64 - sum u_int)),
      // v = 2^16 hi + 2^8 mid + lo (hi, mid: tile nt; lo: tile NT, column nt);
      // 2^8 hi + mid stays below 2^31.
      auto comb = [&](const int (&t)[NT + 1][4], int nt, int row) {
        return fmaf(256.f, (float)(256 * t[nt][2 * row] + t[nt][2 * row + 1]), (float)t[NT][2 * row + nt]);
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
        const float x1 = n1 * (fmaf(cA1[nt], m1, cC1[nt]) + r1 * fmaf(cA2[nt], q1, cC2[nt]));
        const float x2 = n2 * (fmaf(cA1[nt], m2, cC1[nt]) + r2 * fmaf(cA2[nt], q2, cC2[nt]));
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
    ok = __syncthreads_and(okw) != 0;
    if (!ok) break;
    // the key buffer is free: stage the next sub-chunk's keys
    if (tid == 0 && s0 + SC < t_end) issue_keys(s0 + SC);
    // ================= B. weights p ||v||, p = 2^(s - m)
    okw = mbar_wait(bv, phase, P.err);
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
    for (int t = tid; okw && t < scn; t += kThreads) {
      const float vn = s_vn[t];
#pragma unroll
      for (int h4 = 0; h4 < HN; h4 += 4) {
        float4 sc4 = *reinterpret_cast<const float4*>(&s_score[t][h4]);
        float* sc = reinterpret_cast<float*>(&sc4);
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const int h = h4 + hh;
          const float p = h < G ? exp2f(sc[hh] - mnew[h]) : 0.f;
          const float w = p * vn;
          sc[hh] = w;
          lpart[h] += p;
          wmax[h] = fmaxf(wmax[h], w);
        }
        *reinterpret_cast<float4*>(&s_score[t][h4]) = sc4;
      }
    }
#pragma unroll
    for (int h = 0; h < HN; ++h) {
      const float a = warp_sum(lpart[h]), b = warp_max(wmax[h]);
      if (lane == 0) {
        s_red[1][warp][h] = a;
        s_red[2][warp][h] = b;
      }
    }
    ok = __syncthreads_and(okw) != 0;
    if (!ok) break;
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
      float wrow[HN];
#pragma unroll
      for (int h4 = 0; h4 < HN; h4 += 4) {
        const float4 w4 = t < scn ? *reinterpret_cast<const float4*>(&s_score[t][h4]) : make_float4(0.f, 0.f, 0.f, 0.f);
        wrow[h4] = w4.x;
        wrow[h4 + 1] = w4.y;
        wrow[h4 + 2] = w4.z;
        wrow[h4 + 3] = w4.w;
      }
#pragma unroll
      for (int h = 0; h < HN; ++h) {
        if (h < G) {
          const int wi = __float2int_rn(wrow[h] * winv[h]);
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
      corr[nt] = mold == -INFINITY ? 0.f : exp2f(mold - mn);
      wscale[nt] = wi > 0.f ? 1.0f / wi : 0.f;
      int ws = 0;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) ws += __float_as_int(s_red[0][v][h]);
      wtot[nt] = (float)ws;
    }
    // ================= C. values from the staged blocks: coordinates
    // 32 warp + 16 jh + g + 8 row
    int accv[FV][2][NT][4];
#pragma unroll
    for (int f = 0; f < FV; ++f)
#pragma unroll
      for (int jh = 0; jh < 2; ++jh)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) accv[f][jh][nt][0] = accv[f][jh][nt][1] = accv[f][jh][nt][2] = accv[f][jh][nt][3] = 0;
    for (int blk = 0; 32 * blk < scn; ++blk) {
      const uint32_t* vw = s_vc + blk * (KV * DP);
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
          float sv = 0.f;
#pragma unroll
          for (int f = 0; f < FV; ++f)
            sv = fmaf(P.valpha[f], fmaf(256.f, (float)accv[f][jh][nt][2 * rw], (float)accv[f][jh][nt][2 * rw + 1]), sv);
          const float o_sub = wscale[nt] * fmaf(sv, 1.0f / 64.0f, -P.valpha_sum * wtot[nt]);
          o_run[nt][jh][rw] = fmaf(o_run[nt][jh][rw], corr[nt], o_sub);
        }
      }
    }
    __syncthreads();  // every thread has read s_head, s_red, s_wb and the value buffer
    if (tid == 0 && s0 + SC < t_end) issue_values(s0 + SC);
    if (tid < HN && tid < G) {
      float ls = 0.f, mn = 0.f;
#pragma unroll
      for (int v = 0; v < kWarps; ++v) ls += s_red[1][v][tid];
#pragma unroll
      for (int hh = 0; hh < HN; ++hh) mn = hh == tid ? mnew[hh] : mn;
      const float mold = s_head[tid][4];
      const float c = mold == -INFINITY ? 0.f : exp2f(mold - mn);
      s_head[tid][5] = s_head[tid][5] * c + ls;
      s_head[tid][4] = mn;
    }
    __syncthreads();
  }
  if (!ok) {
    // a staging wait expired (error word set): let copies still in flight
    // land, and leave an empty partial (m = -inf: the combine skips it) so
    // that nothing downstream reads stale workspace
    if (tid == 0) {
      mbar_wait(bk, phase, nullptr);
      mbar_wait(bv, phase, nullptr);
    }
    if (tid < G) {
      float* pp = P.part + (((int64_t)grp * P.n_chunks + chunk) * G + tid) * (int64_t)(DP + 2);
      pp[0] = -INFINITY;
      pp[1] = 0.f;
    }
    return;
  }

  // ---- partial (m, l, o_rot) of this chunk (m back in the natural-log domain)
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
      pp[0] = s_head[h][4] * (1.0f / kLog2e);
      pp[1] = s_head[h][5];
    }
  }
}

template <int KK, int KV, int NT, int MQ, int DPT>
cudaError_t launch_nt(const Params& p, dim3 grid, cudaStream_t st) {
  auto kern = attn_kernel<KK, KV, NT, MQ, DPT>;
  const int smem = (int)Layout<KK, KV, NT, MQ, DPT>::bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, DPT, smem, st>>>(p);
  return cudaGetLastError();
}

// d_pad 128 with m = 64 or 128; d_pad 256 with m = 256
template <int KK, int KV>
cudaError_t launch_kv(const Params& p, int m, int dp, dim3 grid, cudaStream_t st) {
  if (dp == 256)
    return p.G <= 4 ? launch_nt<KK, KV, 1, 256, 256>(p, grid, st) : launch_nt<KK, KV, 2, 256, 256>(p, grid, st);
  if (m == 64)
    return p.G <= 4 ? launch_nt<KK, KV, 1, 64, 128>(p, grid, st) : launch_nt<KK, KV, 2, 64, 128>(p, grid, st);
  return p.G <= 4 ? launch_nt<KK, KV, 1, 128, 128>(p, grid, st) : launch_nt<KK, KV, 2, 128, 128>(p, grid, st);
}

template <int KK>
cudaError_t launch_k(const Params& p, int kv, int m, int dp, dim3 grid, cudaStream_t st) {
  switch (kv) {
    case 1: return launch_kv<KK, 1>(p, m, dp, grid, st);
    case 2: return launch_kv<KK, 2>(p, m, dp, grid, st);
    case 3: return launch_kv<KK, 3>(p, m, dp, grid, st);
    case 4: return launch_kv<KK, 4>(p, m, dp, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch(const Params& p, int kk, int kv, int m, int dp, dim3 grid, cudaStream_t st) {
  if (p.G < 1 || p.G > 8) return cudaErrorInvalidValue;
  if (!(dp == 128 && (m == 64 || m == 128)) && !(dp == 256 && m == 256)) return cudaErrorInvalidValue;
  switch (kk) {
    case 1: return launch_k<1>(p, kv, m, dp, grid, st);
    case 2: return launch_k<2>(p, kv, m, dp, grid, st);
    case 3: return launch_k<3>(p, kv, m, dp, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn3
}  // namespace tq
