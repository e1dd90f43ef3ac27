// Scores of many queries against a Q_prod-compressed vector set, and their
// top-k, on the tcgen05 tensor cores (TurboQuant blog notes, unbiased
// inner-product estimator; explainer §8, QJL decoder; turboquant-pytorch
// inner_product / asymmetric_attention_scores; explainer §1, inner-product
// search):
//   s = n ( <q', C[idx]> + kappa rho <u, 2 sigma - 1> ),  q' = Pi q,  u = S q'.
//
// Both inner products are contractions against 0/1 bit matrices (a symmetric
// codebook is an odd function of the index bits: C[idx] = sum over odd
// subsets F of alpha_F (2 b_F - 1), b_F the XOR of the bits in F):
//   <q', C[idx]> = 2 sum_F alpha_F <q', b_F> - sum_F alpha_F sum q',
//   <u, 2 sigma - 1> = 2 <u, sigma> - sum u,
// so the sign part is a popcount-style product of the stored sign bits with
// u.  As an 8-bit MMA: rows (M) are vectors, K the bits, expanded from each
// 32-bit word into eight registers (w >> s) & 0x01010101 (bytes 0 / 1, the K
// order permuted identically on both operands); the other operand holds, per
// query, alpha_F q' (MSE part) or u (sign part) in 24-bit fixed point
// (scale (2^23 - 2^16) / max per query) as three signed balanced bytes in
// three columns.
// Products and sums are exact integers.
//
// The query operands are built once per call (query_scale_kernel, then
// query_digits_kernel), per block of 32 queries: a header with the per-query
// constants and B in chunks of 128 K bytes x 96 rows.  The scoring kernel is
// persistent: a work item is one query block and a range of vectors, in groups
// of two 128-vector tiles that share every B chunk.  Warp 0 stages the B
// chunks with bulk copies (the images stay in L2), warps 1 and 10 issue the
// MMAs of tile 0 and tile 1 (one thread issues one MMA per ~60 cycles, so the
// two tiles get one issuer each), warps 2..9 are the workers: each thread owns
// one vector (one TMEM lane), loads its code words, writes the expanded bits
// to tensor memory with tcgen05.st, and after the group's last chunk folds its
// row of D into 32 scores.  With a top-k requested the scores never leave the
// SM: each query keeps its best k (score descending, index ascending) in
// shared memory, merged per group by one warp per query; the item's lists go
// to the workspace and a final kernel merges the items of each query.  Every
// wait is bounded (error word + clean exit).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "tq_attn_params.h"
#include "tq_device.cuh"
#include "tq_score_tc.h"
#include "tq_wait.cuh"

namespace tq {
namespace score_tc {

constexpr int kQB = 32;              // queries per item
constexpr int kNP = 3 * kQB;         // MMA N per part: 32 queries x 3 digit bytes
constexpr int kRows = 128;           // vectors per tile (MMA M)
constexpr int kGroup = 2 * kRows;    // vectors per group (two tiles)
constexpr int kThreads = 352;        // 11 warps
constexpr int kBStages = 6;
constexpr uint32_t kChunkBytes = 128 * kNP;  // 128 K bytes x 96 rows
constexpr uint32_t kLBO = (kNP / 8) * 128;   // K-direction core-matrix stride of a chunk
constexpr uint32_t kHdr = 512;               // kQB x float4
constexpr int kMaxTopk = 32;
constexpr float kFix = 8323072.0f;           // 2^23 - 2^16: three balanced signed bytes

// TMEM columns: A[buffer][tile] (4 words = 32 columns each), then
// D[tile] = [MSE part 96 | sign part 96]
constexpr uint32_t kTA = 0, kTD = 128, kTDT = 2 * kNP;

// per-thread ring of code words in flight (cp.async): kPD chunks ahead
constexpr int kPD = 8;

// shared memory: B ring | code ring [kPD][kGroup][4 words] | candidate
// scores [kQB][kGroup] | top lists | survivor masks | thresholds | headers
constexpr uint32_t kOffB = 0;
constexpr uint32_t kOffRing = kOffB + kBStages * kChunkBytes;
constexpr uint32_t kOffCand = kOffRing + kPD * kGroup * 16;
constexpr uint32_t kOffTopS = kOffCand + kQB * kGroup * 4;
constexpr uint32_t kOffTopI = kOffTopS + kQB * kMaxTopk * 4;
constexpr uint32_t kOffMask = kOffTopI + kQB * kMaxTopk * 8;  // [kQB][8] survivor bits per warp
constexpr uint32_t kOffThrS = kOffMask + kQB * 8 * 4;          // [kQB] k-th best score
constexpr uint32_t kOffThrI = kOffThrS + kQB * 4;              // [kQB] its index
constexpr uint32_t kOffHdr = kOffThrI + kQB * 8;
constexpr uint32_t kSmem = kOffHdr + 2 * kHdr;

struct Args {
  int wpp, fk, kk, sw;   // words per plane, key features, key code bits, sign words
  int n_mse, n_sgn;      // B chunks of the two parts
  int64_t n_vec, nq;
  const uint32_t* codes;
  const uint32_t* signs;
  const float* norms;
  const float* rnorms;
  int kr16;
  const unsigned char* images;
  uint32_t img_bytes;
  float* scores;
  int topk;
  float* cand_s;     // [items][kQB][topk]
  int64_t* cand_i;
  int64_t groups_per_item, items_per_qb, n_items;
  unsigned* err;
};

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// try_wait parks the polling warp in hardware between tests, which leaves
// the issue slots to the warps doing the work
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, unsigned* err) {
  return bounded_wait<true>(bar, parity, err);
}
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, unsigned* err) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, err)) != 0;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mma_i8(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ uint64_t desc_noswz(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr)
      : "memory");
}

// asynchronous global -> shared copies of 4 or 16 bytes (per thread)
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// (score, index) order of the top-k: score descending, then index ascending
__device__ __forceinline__ bool better(float s1, int64_t i1, float s2, int64_t i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}
__device__ __forceinline__ void warp_best(float& s, int64_t& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const int64_t i2 = __shfl_xor_sync(0xffffffffu, i, o);
    if (better(s2, i2, s, i)) {
      s = s2;
      i = i2;
    }
  }
}
constexpr int64_t kNoIndex = INT64_MAX;

// Feature word f of a k-bit code from its plane words (the planes, then the
// odd triples, in the order of attn::odd_feature_coefs).
__device__ __forceinline__ uint32_t feature_word(const uint32_t* p, int k, int f) {
  if (f < k) return p[f];
  return p[0] ^ p[1] ^ p[2];  // k = 3: the triple {0, 1, 2}
}

// ------------------------------------------------------------------ query operand images

// A word w of the MSE part is feature f = w % fk of plane word cw = w / fk;
// its K slot 4 s + i is coordinate 32 cw + 8 i + s (the bytes of
// (word >> s) & 0x01010101).  Sign part: A word w' is sign word w'.  Row n of
// B = 3 (query) + (digit byte); chunk c of a part holds its K bytes
// [128 c, 128 c + 128) as 8 x 12 core matrices of 8 rows x 16 bytes.
// Per query and part (one warp each): the fixed-point scale inv = kFix /
// max|x| over the part's operand values x (alpha_f q'_j for the MSE part, u_i
// for the signs), stored in qinv, and the header constants of the image,
// which need the integer sum C of the part's rounded values X = rint(x inv):
// x = 2 b - 1 on the code side turns sum_j X_j (2 b_j - 1) into 2 D - C.
__global__ void __launch_bounds__(256) query_scale_kernel(QParams kp, Args a, float kalpha0, float kalpha1,
                                                          float kalpha2, float kalpha3, const float* __restrict__ qrot,
                                                          const float* __restrict__ u, float* __restrict__ qinv,
                                                          unsigned char* __restrict__ img, int64_t n_qb) {
  const int lane = threadIdx.x & 31;
  const int64_t wg = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);  // (query slot, part)
  if (wg >= n_qb * kQB * 2) return;
  const int part = (int)(wg & 1);
  const int64_t qs = wg >> 1, qb = qs / kQB;
  const int ql = (int)(qs % kQB);
  const int dp = kp.d_pad, m = kp.m;
  const float alpha[4] = {kalpha0, kalpha1, kalpha2, kalpha3};
  float amax = 0.f;
  for (int f = 0; f < a.fk; ++f) amax = fmaxf(amax, fabsf(alpha[f]));
  const bool live = qs < a.nq;
  float mx = 0.f;
  if (live) {
    if (part == 0)
      for (int j = lane; j < dp; j += 32) mx = fmaxf(mx, fabsf(qrot[qs * dp + j]));
    else
      for (int j = lane; j < m; j += 32) mx = fmaxf(mx, fabsf(u[qs * m + j]));
  }
  mx = warp_max(mx);
  if (part == 0) mx *= amax;
  const float inv = mx > 0.f ? kFix / mx : 0.f;
  long long C = 0;
  if (live && inv > 0.f) {
    if (part == 0) {
      for (int f = 0; f < a.fk; ++f)
        for (int j = lane; j < dp; j += 32) C += __float2int_rn(alpha[f] * qrot[qs * dp + j] * inv);
    } else {
      for (int j = lane; j < m; j += 32) C += __float2int_rn(u[qs * m + j] * inv);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) C += __shfl_xor_sync(0xffffffffu, C, o);
  if (lane == 0) {
    qinv[qs * 2 + part] = inv;
    float* hdr = reinterpret_cast<float*>(img + qb * (int64_t)a.img_bytes) + 4 * ql + 2 * part;
    const float scale = part == 0 ? 1.0f : kp.kappa;
    hdr[0] = inv > 0.f ? scale * 2.0f / inv : 0.f;
    hdr[1] = inv > 0.f ? (float)(-(double)scale * (double)C / (double)inv) : 0.f;
  }
}

// The B operand of each query block, in chunks of 128 K bytes x 96 rows (row
// n = 3 ql + p holds digit p of query ql's values; K-major core matrices of 8
// rows x 16 bytes).  K byte k of a part's 32-bit word w stands for bit
// 8 (k & 3) + ((k >> 2) & 7) of that word, the order in which the scorer
// expands the code words.  One thread per query and 4 consecutive K bytes.
__global__ void __launch_bounds__(256) query_digits_kernel(QParams kp, Args a, float kalpha0, float kalpha1,
                                                           float kalpha2, float kalpha3,
                                                           const float* __restrict__ qrot,
                                                           const float* __restrict__ u,
                                                           const float* __restrict__ qinv,
                                                           unsigned char* __restrict__ img) {
  const int mse_words = a.fk * a.wpp, kt4 = (mse_words + a.sw) * 8;  // K bytes / 4 per query
  const int64_t qb = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= kQB * kt4) return;
  const int ql = e / kt4, k = 4 * (e % kt4);
  const int64_t q = qb * kQB + ql;
  const int w = k >> 5, s = (k >> 2) & 7;
  const bool sign = w >= mse_words;
  const float alpha[4] = {kalpha0, kalpha1, kalpha2, kalpha3};
  uint32_t dw[3] = {0u, 0u, 0u};
  if (q < a.nq) {
    const float inv = qinv[q * 2 + (sign ? 1 : 0)];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int cc = 8 * i + s;
      float x;
      if (!sign) {
        const int f = w % a.fk, cw = w / a.fk;
        x = alpha[f] * qrot[q * kp.d_pad + 32 * cw + cc] * inv;
      } else {
        x = u[q * kp.m + 32 * (w - mse_words) + cc] * inv;
      }
      const int X = __float2int_rn(x);  // |X| <= 2^23 - 2^16: three balanced signed bytes
      const int d0 = ((X + 128) & 0xFF) - 128, x1 = (X - d0) >> 8;
      const int d1 = ((x1 + 128) & 0xFF) - 128, d2 = (x1 - d1) >> 8;
      dw[0] |= (uint32_t)(d0 & 0xFF) << (8 * i);
      dw[1] |= (uint32_t)(d1 & 0xFF) << (8 * i);
      dw[2] |= (uint32_t)(d2 & 0xFF) << (8 * i);
    }
  }
  const int kp_ = sign ? k - mse_words * 32 : k;  // K byte within the part
  unsigned char* chunk =
      img + qb * (int64_t)a.img_bytes + kHdr + (uint32_t)((sign ? a.n_mse : 0) + (kp_ >> 7)) * kChunkBytes;
  const int kk = kp_ & 127;
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const int n = 3 * ql + p;
    *reinterpret_cast<uint32_t*>(chunk + ((kk >> 4) * (kNP / 8) + (n >> 3)) * 128 + (n & 7) * 16 + (kk & 15)) = dw[p];
  }
}

// ------------------------------------------------------------------ scoring kernel

__global__ void __launch_bounds__(kThreads, 1) score_kernel(Args a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar_bfull[kBStages], bar_bempty[kBStages];
  __shared__ __align__(8) uint64_t bar_afull[2], bar_afree[2], bar_hfull[2], bar_hempty[2];
  __shared__ __align__(8) uint64_t bar_dfull, bar_dempty, bar_wsync, bar_done[2];
  __shared__ uint32_t tmem_base_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto B = [&](uint64_t& b) { return smem_u32(&b); };
  const int nc = a.n_mse + a.n_sgn;
  const int64_t i0 = (int64_t)blockIdx.x * a.n_items / gridDim.x;
  const int64_t i1 = (int64_t)(blockIdx.x + 1) * a.n_items / gridDim.x;
  // vectors of item it: [v0, v1); its groups of two tiles
  auto range = [&](int64_t item, int64_t& v0, int64_t& v1) {
    const int64_t vr = item % a.items_per_qb;
    v0 = vr * a.groups_per_item * kGroup;
    v1 = std::min<int64_t>(a.n_vec, v0 + a.groups_per_item * kGroup);
  };

  if (tid == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(B(bar_bfull[s]), 1);
      mbar_init(B(bar_bempty[s]), 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(B(bar_afull[b]), 8);
      mbar_init(B(bar_afree[b]), 2);
      mbar_init(B(bar_hfull[b]), 1);
      mbar_init(B(bar_hempty[b]), 8);
    }
    mbar_init(B(bar_dfull), 2);
    mbar_init(B(bar_dempty), 8);
    mbar_init(B(bar_wsync), 8);
    mbar_init(B(bar_done[0]), 1);
    mbar_init(B(bar_done[1]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(512u));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  unsigned char* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  const uint32_t s_base = smem_u32(smem);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loader: headers and B chunks
      uint32_t bc = 0;
      int it = 0;
      bool ok = true;
      for (int64_t item = i0; ok && item < i1; ++item, ++it) {
        const int64_t qb = item / a.items_per_qb;
        const unsigned char* img = a.images + qb * (int64_t)a.img_bytes;
        int64_t v0, v1;
        range(item, v0, v1);
        const int64_t groups = (v1 - v0 + kGroup - 1) / kGroup;
        const int ib = it & 1;
        if (it >= 2 && !wait_bar(B(bar_hempty[ib]), ((it - 2) >> 1) & 1, a.err)) break;
        mbar_expect(B(bar_hfull[ib]), kHdr);
        bulk_g2s(s_base + kOffHdr + ib * kHdr, img, kHdr, B(bar_hfull[ib]));
        for (int64_t g = 0; ok && g < groups; ++g) {
          for (int c = 0; c < nc; ++c, ++bc) {
            const int s = bc % kBStages;
            if (bc >= (uint32_t)kBStages && !wait_bar(B(bar_bempty[s]), ((bc / kBStages) - 1) & 1, a.err)) {
              ok = false;
              break;
            }
            mbar_expect(B(bar_bfull[s]), kChunkBytes);
            bulk_g2s(s_base + kOffB + s * kChunkBytes, img + kHdr + (uint32_t)c * kChunkBytes, kChunkBytes,
                     B(bar_bfull[s]));
          }
        }
      }
      for (uint32_t c = bc > (uint32_t)kBStages ? bc - kBStages : 0; c < bc; ++c)
        wait_bar(B(bar_bfull[c % kBStages]), (c / kBStages) & 1, nullptr);
      for (int c = it > 2 ? it - 2 : 0; c < it; ++c) wait_bar(B(bar_hfull[c & 1]), (c >> 1) & 1, nullptr);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 10) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMAs of tile j
      const int j = warp == 1 ? 0 : 1;
      const uint32_t idesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(kNP >> 3) << 17) | ((128u >> 4) << 24);
      uint32_t cc = 0, gc = 0;
      bool ok = true;
      for (int64_t item = i0; ok && item < i1; ++item) {
        int64_t v0, v1;
        range(item, v0, v1);
        const int64_t groups = (v1 - v0 + kGroup - 1) / kGroup;
        for (int64_t g = 0; ok && g < groups; ++g, ++gc) {
          for (int c = 0; c < nc; ++c, ++cc) {
            const uint32_t buf = cc & 1, s = cc % kBStages;
            if (!wait_bar(B(bar_afull[buf]), (cc >> 1) & 1, a.err) ||
                !wait_bar(B(bar_bfull[s]), (cc / kBStages) & 1, a.err) ||
                (c == 0 && gc >= 1 && !wait_bar(B(bar_dempty), (gc - 1) & 1, a.err))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int part = c < a.n_mse ? 0 : 1;
            const bool first = c == 0 || c == a.n_mse;
            const uint32_t d = tmem + kTD + (uint32_t)(j * kTDT + part * kNP);
            const uint32_t av = tmem + kTA + (buf * 2 + j) * 32;
            const uint64_t bd = desc_noswz(s_base + kOffB + s * kChunkBytes, kLBO, 128);
#pragma unroll
            for (int t = 0; t < 4; ++t)
              mma_i8(d, av + 8 * t, bd + (uint64_t)((t * 2 * kLBO) >> 4), idesc, (first && t == 0) ? 0u : 1u);
            tc_commit(B(bar_afree[buf]));
            tc_commit(B(bar_bempty[s]));
          }
          if (ok) tc_commit(B(bar_dfull));
        }
      }
      tc_commit(B(bar_done[j]));
      wait_bar(B(bar_done[j]), 0, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- workers: one vector each
    const int tile = (warp - 2) >> 2, q4 = warp & 3;
    const int row = 32 * q4 + lane;
    const int t_id = tile * kRows + row;  // 0..255 within the group
    const int wsel = warp - 2;            // selection warp index 0..7
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const int KW = a.kk * a.wpp;
    float* cand = reinterpret_cast<float*>(smem + kOffCand);       // [kQB][kGroup]
    float* top_s = reinterpret_cast<float*>(smem + kOffTopS);      // [kQB][kMaxTopk]
    int64_t* top_i = reinterpret_cast<int64_t*>(smem + kOffTopI);  // [kQB][kMaxTopk]
    uint32_t* smask = reinterpret_cast<uint32_t*>(smem + kOffMask);   // [kQB][8]
    float* thr_s = reinterpret_cast<float*>(smem + kOffThrS);         // [kQB]
    int64_t* thr_i = reinterpret_cast<int64_t*>(smem + kOffThrI);     // [kQB]
    const int K = a.topk;
    int64_t prev_qb = -1;
    uint32_t cc = 0, gc = 0, ws = 0;
    int it = 0;
    bool ok = true;
    auto wsync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(B(bar_wsync));
      const bool r_ok = wait_bar_warp(B(bar_wsync), ws & 1, a.err);
      ++ws;
      return r_ok;
    };
    // The raw words of chunk c of vector v go to ring slot c % kPD: the sign
    // words, or the plane words that make its four feature words (fk = 1: 4
    // plane words; fk = 2: planes 0, 1 of 2 plane-word positions; fk = 4:
    // planes 0..2 of one position).
    const uint32_t ring = s_base + kOffRing + (uint32_t)t_id * 16;
    auto issue_chunk = [&](int64_t v, int c) {
      const uint32_t dst = ring + (uint32_t)(c % kPD) * (kGroup * 16);
      if (c >= a.n_mse) {
        cp_async16(dst, a.signs + v * a.sw + 4 * (c - a.n_mse));
        return;
      }
      const uint32_t* rw = a.codes + v * KW;
      if (a.fk == 1) {
        cp_async16(dst, rw + 4 * c);
      } else if (a.fk == 2) {
        cp_async8(dst, rw + 2 * c);
        cp_async8(dst + 8, rw + a.wpp + 2 * c);
      } else {
        cp_async4(dst, rw + c);
        cp_async4(dst + 4, rw + a.wpp + c);
        cp_async4(dst + 8, rw + 2 * a.wpp + c);
      }
    };
    // the four A words of chunk c (in order: feature f of position cw at
    // 4 c + i = cw fk + f) from its ring slot
    auto read_chunk = [&](int c, uint32_t (&w)[4]) {
      const uint4 r = *reinterpret_cast<const uint4*>(smem + kOffRing + (c % kPD) * (kGroup * 16) + t_id * 16);
      if (c >= a.n_mse || a.fk == 1) {
        w[0] = r.x; w[1] = r.y; w[2] = r.z; w[3] = r.w;
      } else if (a.fk == 2) {  // r = plane 0 of (cw0, cw1), plane 1 of (cw0, cw1)
        w[0] = r.x; w[1] = r.z; w[2] = r.y; w[3] = r.w;
      } else {                 // r = planes 0, 1, 2 of one position
        w[0] = r.x; w[1] = r.y; w[2] = r.z; w[3] = r.x ^ r.y ^ r.z;
      }
    };
    for (int64_t item = i0; ok && item < i1; ++item, ++it) {
      const int64_t qb = item / a.items_per_qb;
      int64_t v0, v1;
      range(item, v0, v1);
      const int64_t groups = (v1 - v0 + kGroup - 1) / kGroup;
      const int ib = it & 1;
      if (!wait_bar_warp(B(bar_hfull[ib]), (it >> 1) & 1, a.err)) { ok = false; break; }
      const float4* hdr = reinterpret_cast<const float4*>(smem + kOffHdr + ib * kHdr);
      // The lists carry over between consecutive items of one query block: an
      // item's list then also holds earlier ranges' entries (the final merge
      // skips repeats), and the carried k-th best filters this range early.
      if (K > 0 && qb != prev_qb) {
        for (int e = t_id; e < kQB * kMaxTopk; e += kGroup) {
          top_s[e] = -INFINITY;
          top_i[e] = kNoIndex;
        }
        if (t_id < kQB) {
          thr_s[t_id] = -INFINITY;
          thr_i[t_id] = kNoIndex;
        }
        if (!wsync()) { ok = false; break; }
      }
      prev_qb = qb;
      for (int64_t g = 0; ok && g < groups; ++g, ++gc) {
        const int64_t v = v0 + g * kGroup + t_id;
        const bool valid = v < v1;
        // kPD chunks in flight (one copy group per chunk, empty past the end)
        for (int c = 0; c < kPD; ++c) {
          if (valid && c < nc) issue_chunk(v, c);
          cp_commit();
        }
        for (int c = 0; c < nc; ++c, ++cc) {
          const uint32_t buf = cc & 1;
          uint32_t wcur[4] = {0u, 0u, 0u, 0u};
          cp_wait<kPD - 1>();  // chunk c's copies have landed
          if (valid) read_chunk(c, wcur);
          __syncwarp();        // the slot's reads are done before it is refilled
          if (valid && c + kPD < nc) issue_chunk(v, c + kPD);
          cp_commit();
          if (cc >= 2 && !wait_bar_warp(B(bar_afree[buf]), ((cc - 2) >> 1) & 1, a.err)) { ok = false; break; }
          uint32_t reg[32];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int s = 0; s < 8; ++s) reg[8 * i + s] = (wcur[i] >> s) & 0x01010101u;
          tmem_st32(tmem + kTA + (buf * 2 + tile) * 32 + lane_off, reg);
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(B(bar_afull[buf]));
        }
        cp_wait<0>();  // nothing of this group stays in flight (error exit)
        if (!ok) break;
        // ---- the group's scores
        if (!wait_bar_warp(B(bar_dfull), gc & 1, a.err)) { ok = false; break; }
        tc_fence_after();
        const float n = valid ? a.norms[v] : 0.f;
        const float rho = valid ? get_rnorm(a.rnorms, v, a.kr16) : 0.f;
        // two halves of 16 queries: 48 MSE and 48 sign columns each
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t dm[48], ds[48];
          const uint32_t col = tmem + kTD + tile * kTDT + 48 * half + lane_off;
          tmem_ld32(col, dm);
          tmem_ld16(col + 32, dm + 32);
          tmem_ld32(col + kNP, ds);
          tmem_ld16(col + kNP + 32, ds + 32);
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(B(bar_dempty));
          }
#pragma unroll
          for (int qq = 0; qq < 16; ++qq) {
            const int ql = 16 * half + qq;
            const int64_t q = qb * kQB + ql;
            const float4 c4 = hdr[ql];
            auto comb = [&](const uint32_t* d3) {
              const float v = fmaf((float)(int)d3[2], 256.f, (float)(int)d3[1]);
              return fmaf(v, 256.f, (float)(int)d3[0]);
            };
            const float Dm = comb(dm + 3 * qq), Ds = comb(ds + 3 * qq);
            const float sc = n * fmaf(rho, fmaf(c4.z, Ds, c4.w), fmaf(c4.x, Dm, c4.y));
            if (a.scores && valid && q < a.nq) a.scores[q * a.n_vec + v] = sc;
            if (K > 0) {
              // survivors: valid vectors ahead of the query's current k-th best
              const bool sv = valid && better(sc, v, thr_s[ql], thr_i[ql]);
              const uint32_t bits = __ballot_sync(0xffffffffu, sv);
              if (sv) cand[ql * kGroup + t_id] = sc;
              if (lane == 0) smask[ql * 8 + (t_id >> 5)] = bits;  // word = the warp's 32-vector block
            }
          }
        }
        if (K == 0) continue;
        // ---- merge the group's candidates into each query's best K (one
        // warp per query)
        if (!wsync()) { ok = false; break; }
        const int64_t gbase = v0 + g * kGroup;
        for (int ql = wsel; ql < kQB; ql += 8) {
          float* ts = top_s + ql * kMaxTopk;
          int64_t* ti = top_i + ql * kMaxTopk;
          const uint32_t mw = lane < 8 ? smask[ql * 8 + lane] : 0u;
          const int nsurv = __reduce_add_sync(0xffffffffu, (unsigned)__popc(mw));
          if (nsurv == 0) continue;
          // the list, lane r < K holding rank r
          float ls = lane < K ? ts[lane] : -INFINITY;
          int64_t li = lane < K ? ti[lane] : kNoIndex;
          if (nsurv <= 24) {
            // few survivors: insert each one that still beats the k-th best
            float ks = __shfl_sync(0xffffffffu, ls, K - 1);
            int64_t ki = __shfl_sync(0xffffffffu, li, K - 1);
            for (int w8 = 0; w8 < 8; ++w8) {
              uint32_t bits = __shfl_sync(0xffffffffu, mw, w8);
              while (bits) {
                const int t = 32 * w8 + __ffs(bits) - 1;
                bits &= bits - 1;
                const float cs = cand[ql * kGroup + t];
                const int64_t ci = gbase + t;
                if (!better(cs, ci, ks, ki)) continue;
                const int pos = __popc(__ballot_sync(0xffffffffu, lane < K && better(ls, li, cs, ci)));
                const float us = __shfl_up_sync(0xffffffffu, ls, 1);
                const int64_t ui = __shfl_up_sync(0xffffffffu, li, 1);
                if (lane == pos) {
                  ls = cs;
                  li = ci;
                } else if (lane > pos) {
                  ls = us;
                  li = ui;
                }
                ks = __shfl_sync(0xffffffffu, ls, K - 1);
                ki = __shfl_sync(0xffffffffu, li, K - 1);
              }
            }
          } else {
            // many survivors: K rounds of the warp's best over the survivors
            // (8 per lane) and the list
            float cs[9];
            int64_t ci[9];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int t = lane + 32 * e;
              const bool sv = (__shfl_sync(0xffffffffu, mw, e) >> lane) & 1u;
              cs[e] = sv ? cand[ql * kGroup + t] : -INFINITY;
              ci[e] = sv ? gbase + t : kNoIndex;
            }
            cs[8] = ls;
            ci[8] = li;
            for (int r = 0; r < K; ++r) {
              float bs = -INFINITY;
              int64_t bi = kNoIndex;
#pragma unroll
              for (int e = 0; e < 9; ++e)
                if (better(cs[e], ci[e], bs, bi)) {
                  bs = cs[e];
                  bi = ci[e];
                }
              warp_best(bs, bi);
#pragma unroll
              for (int e = 0; e < 9; ++e)
                if (ci[e] == bi && cs[e] == bs) {
                  cs[e] = -INFINITY;
                  ci[e] = kNoIndex;
                }
              if (lane == r) {
                ls = bs;
                li = bi;
              }
            }
          }
          if (lane < K) {
            ts[lane] = ls;
            ti[lane] = li;
          }
          if (lane == K - 1) {
            thr_s[ql] = ls;
            thr_i[ql] = li;
          }
          __syncwarp();
        }
        if (!wsync()) { ok = false; break; }  // the candidate buffer is reused by the next group
      }
      if (!ok) break;
      if (K > 0) {
        const int64_t base = item * kQB * K;
        for (int e = t_id; e < kQB * K; e += kGroup) {
          const int ql = e / K, r = e % K;
          a.cand_s[base + e] = top_s[ql * kMaxTopk + r];
          a.cand_i[base + e] = top_i[ql * kMaxTopk + r];
        }
        if (!wsync()) { ok = false; break; }  // the next item resets or extends the lists
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(B(bar_hempty[ib]));
    }
    if (!ok && K > 0) {
      // a wait expired (error word set): the unfinished items offer no candidates
      for (int64_t item = i0 + it; item < i1; ++item)
        for (int e = t_id; e < kQB * K; e += kGroup) {
          a.cand_s[item * kQB * K + e] = -INFINITY;
          a.cand_i[item * kQB * K + e] = kNoIndex;
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u));
  }
}

// Final top-k of each query over its items' lists (one warp per query):
// K rounds, each picking the best candidate strictly after the previous pick
// in the (score descending, index ascending) order.
__global__ void __launch_bounds__(128) merge_kernel(const float* __restrict__ cand_s,
                                                   const int64_t* __restrict__ cand_i, int64_t nq,
                                                   int64_t items_per_qb, int K, float* __restrict__ top_s,
                                                   int64_t* __restrict__ top_i) {
  const int lane = threadIdx.x & 31;
  const int64_t q = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (q >= nq) return;
  const int64_t qb = q / kQB, ql = q % kQB;
  const int64_t n = items_per_qb * K;
  float ps = INFINITY;
  int64_t pi = -1;  // previous pick (starts before every candidate)
  for (int r = 0; r < K; ++r) {
    float bs = -INFINITY;
    int64_t bi = kNoIndex;
    for (int64_t e = lane; e < n; e += 32) {
      const int64_t item = qb * items_per_qb + e / K;
      const int64_t o = (item * kQB + ql) * K + e % K;
      const float s = cand_s[o];
      const int64_t i = cand_i[o];
      if (i != kNoIndex && better(ps, pi, s, i) && better(s, i, bs, bi)) {
        bs = s;
        bi = i;
      }
    }
    warp_best(bs, bi);
    if (lane == 0) {
      top_s[q * K + r] = bs;
      top_i[q * K + r] = bi;
    }
    ps = bs;
    pi = bi;
  }
}

// ------------------------------------------------------------------ host side

namespace {
Args make_args(const QParams& kp, int64_t nq, int64_t n_vec, int topk, int num_sms) {
  Args a{};
  a.wpp = kp.d_pad / 32;
  a.kk = kp.k;
  a.fk = 1 << (kp.k - 1);
  a.sw = kp.m / 32;
  a.n_mse = a.fk * a.wpp / 4;
  a.n_sgn = a.sw / 4;
  a.n_vec = n_vec;
  a.nq = nq;
  a.img_bytes = kHdr + (uint32_t)(a.n_mse + a.n_sgn) * kChunkBytes;
  a.topk = topk;
  const int64_t n_qb = (nq + kQB - 1) / kQB;
  const int64_t n_groups = (n_vec + kGroup - 1) / kGroup;
  // about four items per SM (rounded so items stay whole groups)
  const int64_t want = std::max<int64_t>(1, (int64_t)num_sms * 4 / std::max<int64_t>(n_qb, 1));
  a.items_per_qb = std::min<int64_t>(want, n_groups);
  a.groups_per_item = (n_groups + a.items_per_qb - 1) / a.items_per_qb;
  a.items_per_qb = (n_groups + a.groups_per_item - 1) / a.groups_per_item;
  a.n_items = n_qb * a.items_per_qb;
  return a;
}
inline size_t up256(size_t v) { return (v + 255) / 256 * 256; }
}  // namespace

bool covers(const QParams& kp, int topk) {
  if (kp.k < 1 || kp.k > 3 || kp.m <= 0 || kp.m % 128 != 0 || kp.d_pad % 32 != 0) return false;
  const int fk = 1 << (kp.k - 1), wpp = kp.d_pad / 32;
  return (fk * wpp) % 4 == 0 && topk <= kMaxTopk;
}

size_t workspace_bytes(const QParams& kp, int64_t nq, int64_t n_vec, int topk) {
  const Args a = make_args(kp, nq, n_vec, topk, 148);
  const int64_t n_qb = (nq + kQB - 1) / kQB;
  // the item count depends on the SM count: size the candidates for up to
  // 4 x 1024 items per query block
  const int64_t items_max = n_qb * std::min<int64_t>((n_vec + kGroup - 1) / kGroup, 4096);
  size_t b = up256((size_t)n_qb * a.img_bytes) + up256((size_t)n_qb * kQB * 2 * 4);
  if (topk > 0) b += up256((size_t)items_max * kQB * topk * 4) + up256((size_t)items_max * kQB * topk * 8);
  return b;
}

cudaError_t launch(const QParams& kp, const float* qrot, const float* u, int64_t nq, const uint32_t* codes,
                   const uint32_t* signs, const float* norms, const float* rnorms, int64_t n_vec, float* scores,
                   int topk, float* top_s, int64_t* top_i, void* ws, unsigned* err, int num_sms, cudaStream_t st) {
  if (!covers(kp, topk)) return cudaErrorInvalidValue;
  Args a = make_args(kp, nq, n_vec, topk, num_sms);
  const int64_t n_qb = (nq + kQB - 1) / kQB;
  unsigned char* w = (unsigned char*)ws;
  unsigned char* images = w;
  w += up256((size_t)n_qb * a.img_bytes);
  float* qinv = (float*)w;
  w += up256((size_t)n_qb * kQB * 2 * 4);
  a.codes = codes;
  a.signs = signs;
  a.norms = norms;
  a.rnorms = rnorms;
  a.kr16 = kp.rnorm_f16;
  a.images = images;
  a.scores = scores;
  a.err = err;
  if (topk > 0) {
    const int64_t items_max = n_qb * std::min<int64_t>((n_vec + kGroup - 1) / kGroup, 4096);
    if (a.n_items > items_max) return cudaErrorInvalidValue;
    a.cand_s = (float*)w;
    w += up256((size_t)items_max * kQB * topk * 4);
    a.cand_i = (int64_t*)w;
  }
  float alpha[8], asum;
  attn::odd_feature_coefs(kp.centroids, kp.k, alpha, &asum);
  query_scale_kernel<<<(unsigned)((n_qb * kQB * 2 + 7) / 8), 256, 0, st>>>(kp, a, alpha[0], alpha[1], alpha[2],
                                                                             alpha[3], qrot, u, qinv, images, n_qb);
  const int kt4 = (a.fk * a.wpp + a.sw) * 8;
  query_digits_kernel<<<dim3((unsigned)((kQB * kt4 + 255) / 256), (unsigned)n_qb), 256, 0, st>>>(
      kp, a, alpha[0], alpha[1], alpha[2], alpha[3], qrot, u, qinv, images);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // one CTA per SM (it allocates all 512 TMEM columns): the shared memory
  // request keeps a second CTA off the SM
  const uint32_t smem = std::max<uint32_t>(kSmem + 128, 116 * 1024);
  e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t ctas = std::min<int64_t>(a.n_items, num_sms);
  score_kernel<<<(unsigned)ctas, kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || topk == 0) return e;
  merge_kernel<<<(unsigned)((nq + 3) / 4), 128, 0, st>>>(a.cand_s, a.cand_i, nq, a.items_per_qb, topk, top_s, top_i);
  return cudaGetLastError();
}

}  // namespace score_tc
}  // namespace tq
