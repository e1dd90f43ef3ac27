// Encode kernels with the rotation on the tensor cores (d_pad = 128, fp16 or
// bf16 input, randomized Hadamard rotation).
//
// Same method as the other encoders (TurboQuant blog notes, Q_MSE and the
// definition of Q_prod; explainer §6, §8): n = ||x||, y = H D x / (sqrt(d_pad) n),
// idx = #{k : B_k < y}, bit-packed codes; Q_prod adds r = y - C[idx],
// rho = ||r|| and the sign bits of S r.
//
// The randomized Hadamard rotation is the product with the d_pad x d_pad
// matrix H D, whose entries are +-1: exact in fp16 and bf16.  One tcgen05 MMA
// per tile of 128 vectors computes u = (H D) x for all of them with exact
// products and fp32 accumulation, so the CUDA cores are left with the
// per-coordinate quantization only.  Roles inside a persistent CTA (one per SM):
//   warp 0      TMA producer: tiles of 128 consecutive input rows, two
//               128-byte-swizzled boxes of 64 columns each, into a 4-stage ring;
//   warp 1      TMEM allocator and MMA issuer (one elected thread);
//   the rest    the epilogue, reading u from TMEM (warp w may read TMEM lanes
//               32 (w % 4) .. +31, i.e. those vectors of the tile).
// Q_MSE (encode_tc_kernel): two epilogue groups of four warps, group g owns
// TMEM buffer g and every second tile; one thread per vector computes
// n = ||u|| / sqrt(d_pad) and the bit planes (sign plane and thermometer
// planes of |u| against the positive boundaries scaled by ||u||).
// Q_prod (encode_prod_rows_kernel): the same two groups and one thread per
// vector; the epilogue writes r = u / ||u|| - C[idx] (times 2^10, split into
// fp16 hi + lo parts) back over u, a second MMA forms S r (A = r from TMEM,
// B = S from shared memory), and the group packs the QJL sign words of its
// rows while the other group quantizes the next tile.
// Exact boundary ties on the negative side resolve toward zero here (the
// oracle resolves them to the lower cell); such values lie inside the parity
// window by definition.
//
// Requirements checked by the host: rows are 16-byte aligned (d * 2 and the
// row stride multiples of 16 bytes), every segment holds a multiple of 32
// vectors (so each warp's 32 rows are one BLOCK32 block of one segment), and
// m <= 128 for Q_prod.  Every wait is bounded; on expiry the device error word
// is set and the CTA winds down.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "tq_device.cuh"
#include "tq_enc3.h"
#include "tq_wait.cuh"

namespace tq {
namespace enc3 {

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Bounded wait for the phase with the given parity (try_wait, which parks
// the polling warp between tests and leaves its issue slots to the working
// warps; measured slightly faster here than non-blocking polls): false, and
// the device error word set, if it has not completed within the wait budget.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* err) {
  return bounded_wait<true>(bar, parity, err);
}

// Warp-uniform form: every lane waits, the warp proceeds only if all saw it.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, unsigned* err) {
  const bool ok = mbar_wait(bar, parity, err);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D (TMEM) (+)= A (smem descriptor) * B (smem descriptor)^T
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc));
}
// D (TMEM) (+)= A (TMEM) * B (smem descriptor)^T
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc));
}

// Shared-memory matrix descriptors (K-major operands).
//  * no swizzle: 8x8 core matrices of 128 contiguous bytes, LBO = stride between
//    core matrices along K, SBO = stride between 8-row groups;
//  * 128-byte swizzle (what TMA writes for a box 64 x 16-bit wide): rows of
//    128 bytes, 8-row groups 1024 bytes apart, chunks XOR-permuted by row.
__device__ __forceinline__ uint64_t desc_noswz(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Byte offset of element (row, k) in a no-swizzle K-major tile of `rows` rows.
__device__ __forceinline__ uint32_t core_offset(int row, int k, int rows) {
  return (uint32_t)(((k >> 3) * (rows >> 3) + (row >> 3)) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}

// tcgen05.ld of 32 columns and its completion in one statement: the
// registers are defined only once the data has arrived.
__device__ __forceinline__ void tmem_ld32_sync(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr)
      : "memory");
}

// Packed pairs of fp32 (the f32x2 forms of add, sub and fma).
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 upk2(uint64_t r) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(r));
  return f;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// Complete the outstanding tcgen05.ld of this thread; the empty asm
// statements keep every use of the loaded registers after the wait.
__device__ __forceinline__ void tmem_ld_wait1(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}
__device__ __forceinline__ void tmem_ld_wait2(uint32_t (&r)[32], uint32_t (&q)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]), "+r"(q[i]));
}

__device__ __forceinline__ void tmem_st8(uint32_t addr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(addr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// ------------------------------------------------------------------ quantize + pack

// 0xFFFFFFFF if a > b else 0 (an integer mask instead of a predicate).
__device__ __forceinline__ uint32_t gt_mask(float a, float b) {
  uint32_t r;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(a), "f"(b));
  return r;
}
// m ? a : b for an all-ones / all-zeros mask m
__device__ __forceinline__ float sel_mask(uint32_t m, float a, float b) {
  return __uint_as_float((m & __float_as_uint(a)) | (~m & __float_as_uint(b)));
}

// Sign bit of a - b.  The sign of a rounded difference is the sign of the
// exact one and equal operands give +0, so for b = |u| and a = t the bit is
// exactly [|u| > t]; for a = 0 and b = u it is [u > 0].
__device__ __forceinline__ uint32_t sub_bits(float a, float b) {
  float r;
  asm("sub.rn.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return __float_as_uint(r);
}
// w << 1 with the sign bit of v shifted in at bit 0
__device__ __forceinline__ uint32_t shift_in(uint32_t w, uint32_t v) { return __funnelshift_l(v, w, 1); }
// 1.0 if v < 0 else 0.0, for |v| >= 2^-40 or v = +0
__device__ __forceinline__ float step_neg(float v) {
  float r;
  asm("mul.rn.sat.f32 %0, %1, 0fD3800000;" : "=f"(r) : "f"(v));  // v * -2^40, clamped to [0, 1]
  return r;
}

// Planes of idx = s ? 2^(K-1) + mu : 2^(K-1) - 1 - mu from the sign plane S
// and the magnitude bits M of mu: the top plane is S, the lower ones ~(S ^ M).
template <int K>
__device__ __forceinline__ void planes_from(uint32_t S, uint32_t M0, uint32_t M1, uint32_t M2,
                                            uint32_t (&plane)[K]) {
  plane[K - 1] = S;
  if (K >= 2) plane[0] = ~(S ^ M0);
  if (K >= 3) plane[1] = ~(S ^ M1);
  if (K >= 4) plane[2] = ~(S ^ M2);
}

// |C[idx]| of one coordinate from a = |u| and the positive thresholds t,
// taking the same decisions as quant32_mse (thermometer for K <= 3, binary
// search for K = 4); cp = the positive centroids (unit domain).
template <int K>
__device__ __forceinline__ float mag_centroid(float a, const float (&t)[8], const float (&cp)[8]) {
  if (K == 1) return cp[0];
  if (K == 2) return a > t[0] ? cp[1] : cp[0];
  if (K == 3) return a > t[1] ? (a > t[2] ? cp[3] : cp[2]) : (a > t[0] ? cp[1] : cp[0]);
  const bool m2 = a > t[3];
  const bool m1 = a > (m2 ? t[5] : t[1]);
  const bool m0 = a > (m1 ? (m2 ? t[6] : t[2]) : (m2 ? t[4] : t[0]));
  return m2 ? (m1 ? (m0 ? cp[7] : cp[6]) : (m0 ? cp[5] : cp[4]))
            : (m1 ? (m0 ? cp[3] : cp[2]) : (m0 ? cp[1] : cp[0]));
}

// Q_MSE quantization of 32 coordinates u[0..32) (coordinate 32c + i in u[i])
// against the positive thresholds t (boundaries times ||u||), bit planes
// shifted into words (bit i = coordinate 32c + i).  K <= 3: every threshold
// gives one thermometer plane T_j = [|u| > t_j]; the magnitude index
// mu = T_0 + T_1 + T_2 has bits M1 = T_1 and M0 = T_0 ^ T_1 ^ T_2.  Each bit
// costs one subtraction and one funnel shift.  K = 4: binary search of |u|
// with integer masks.
// DOT (K <= 3): dot += sum |u| |C[idx]| from the thermometer, with cp the
// positive centroids: |C| = cp_0 + sum_j T_j (cp_(j+1) - cp_j), and over the
// 32 coordinates sum_{|u| > t_j} |u| = t_j popc(T_j) + sum max(|u| - t_j, 0),
// where sum max(|u| - t, 0) = (sum |u| - 32 t + sum |t - |u||) / 2 needs one
// addition per coordinate and threshold.  K = 4 selects |C| per coordinate.
template <int K, bool DOT = false>
__device__ __forceinline__ void quant32_mse(const uint32_t (&ur)[32], const float (&t)[8],
                                            uint32_t (&plane)[K], const float (&cp)[8], float& dot) {
  uint32_t S = 0, M0 = 0, M1 = 0, M2 = 0;
  if (K <= 3) {
    uint32_t T0 = 0, T1 = 0, T2 = 0;
    float sa = 0.f, D0 = 0.f, D1 = 0.f, D2 = 0.f;  // sum |u|, sum |t_j - |u||
#pragma unroll
    for (int i = 31; i >= 0; --i) {
      const float u = __uint_as_float(ur[i]);
      const float a = fabsf(u);
      S = shift_in(S, sub_bits(0.0f, u));
      if (DOT) sa += a;
      // DOT: the differences in plain C, so that |u| and |d| fold into the
      // additions as operand modifiers (same rounding as sub_bits)
      if (K >= 2) {
        uint32_t d0;
        if (DOT) {
          const float f = t[0] - a;
          d0 = __float_as_uint(f);
          D0 += fabsf(f);
        } else {
          d0 = sub_bits(t[0], a);
        }
        T0 = shift_in(T0, d0);
      }
      if (K >= 3) {
        uint32_t d1, d2;
        if (DOT) {
          const float f1 = t[1] - a, f2 = t[2] - a;
          d1 = __float_as_uint(f1);
          d2 = __float_as_uint(f2);
          D1 += fabsf(f1);
          D2 += fabsf(f2);
        } else {
          d1 = sub_bits(t[1], a);
          d2 = sub_bits(t[2], a);
        }
        T1 = shift_in(T1, d1);
        T2 = shift_in(T2, d2);
      }
    }
    M0 = K == 3 ? (T0 ^ T1 ^ T2) : T0;
    M1 = T1;
    if (DOT) {
      // sum over |u| > t of |u|
      auto above = [&](float tj, uint32_t Tj, float Dj) {
        return fmaf(tj, (float)__popc(Tj), 0.5f * (sa + fmaf(-32.0f, tj, Dj)));
      };
      float acc = cp[0] * sa;
      if (K >= 2) acc = fmaf(cp[1] - cp[0], above(t[0], T0, D0), acc);
      if (K >= 3) {
        acc = fmaf(cp[2] - cp[1], above(t[1], T1, D1), acc);
        acc = fmaf(cp[3] - cp[2], above(t[2], T2, D2), acc);
      }
      dot += acc;
    }
  } else {
#pragma unroll
    for (int i = 31; i >= 0; --i) {
      const float u = __uint_as_float(ur[i]);
      const float a = fabsf(u);
      S = shift_in(S, sub_bits(0.0f, u));
      const uint32_t m2 = gt_mask(a, t[3]);
      const uint32_t m1 = gt_mask(a, sel_mask(m2, t[5], t[1]));
      const float tA = sel_mask(m2, t[6], t[2]), tB = sel_mask(m2, t[4], t[0]);
      const uint32_t m0 = gt_mask(a, sel_mask(m1, tA, tB));
      M2 = M2 + M2 - m2;
      M1 = M1 + M1 - m1;
      M0 = M0 + M0 - m0;
      if (DOT) dot = fmaf(a, mag_centroid<K>(a, t, cp), dot);
    }
  }
  planes_from<K>(S, M0, M1, M2, plane);
}

// Q_prod's MSE stage (K <= 3 bits) for 32 coordinates, in the scaled unit
// domain a' = |u| * inv with inv = 2^10 / ||u||: thresholds T_j = 2^10 t_j and
// magnitudes C_j = 2^10 c_j (tc[j] = T_j - C_0, dc[j] = C_(j+1) - C_j).  With
// e0 = a' - C_0 and d_j = T_j - a', the thermometer bit is sign(d_j), the step
// [d_j < 0] is exact in {0, 1}, and e = e0 - sum_j step_j dc_j = a' - C_mu.
// v[i] becomes 2^10 r = +-e with the sign of the coordinate (r = y - C[idx]).
// The sign plane comes from the sign bits of u:
// NS (bit set = negative) is shifted in and S = ~NS per word.
// An exactly zero coordinate of a nonzero vector then takes the upper middle
// cell (a tie at the middle boundary, y = 0 = B); the caller forces S = 0 for
// zero vectors.  The residual keeps the coordinate's sign bit.
template <int K>
__device__ __forceinline__ void quant32_prod_sb(float (&v)[32], const float (&tc)[4], const float (&dc)[4],
                                                float c0, float inv, uint32_t& NS, uint32_t& T0,
                                                uint32_t& T1, uint32_t& T2) {
#pragma unroll
  for (int i = 31; i >= 0; --i) {
    const uint32_t ub = __float_as_uint(v[i]);
    NS = shift_in(NS, ub);
    const float e0 = fmaf(fabsf(v[i]), inv, -c0);
    float e = e0;
    if (K >= 2) {
      const float d0 = tc[0] - e0;
      T0 = shift_in(T0, __float_as_uint(d0));
      e = fmaf(step_neg(d0), -dc[0], e);
      if (K >= 3) {
        const float d1 = tc[1] - e0, d2 = tc[2] - e0;
        T1 = shift_in(T1, __float_as_uint(d1));
        T2 = shift_in(T2, __float_as_uint(d2));
        e = fmaf(step_neg(d1), -dc[1], e);
        e = fmaf(step_neg(d2), -dc[2], e);
      }
    }
    v[i] = __uint_as_float(__float_as_uint(e) ^ (ub & 0x80000000u));
  }
}

// 32x32 bit transpose across the warp: lane t holds row t (bit i); returns
// column `lane` (bit t = row t's bit `lane`).
struct TransposeCtl {
  uint32_t keep[5];
  uint32_t amt[5];
};

__device__ __forceinline__ TransposeCtl make_transpose_ctl(int lane) {
  const uint32_t low[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
  TransposeCtl c;
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int s = 16 >> r;
    const bool hi = (lane & s) != 0;
    c.keep[r] = hi ? ~low[r] : low[r];
    c.amt[r] = hi ? (uint32_t)(32 - s) : (uint32_t)s;
  }
  return c;
}

__device__ __forceinline__ uint32_t transpose32(uint32_t w, const TransposeCtl& c) {
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int s = 16 >> r;
    const uint32_t o = __shfl_xor_sync(0xffffffffu, w, s);
    const uint32_t rot = __funnelshift_l(o, o, c.amt[r]);
    w = (w & c.keep[r]) | (rot & ~c.keep[r]);
  }
  return w;
}

// ------------------------------------------------------------------ kernel

template <typename T, int K, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap xmap, QParams qp, Args a) {
  constexpr bool BLOCK = MODE == MODE_MSE_BLOCK || MODE == MODE_MSE_BLOCK_U;
  constexpr bool UNB = MODE == MODE_MSE_ROW_U || MODE == MODE_MSE_BLOCK_U;  // EDEN scale
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStages], bar_empty[kStages];
  __shared__ __align__(8) uint64_t bar_accf[2], bar_acce[2], bar_done;
  __shared__ uint32_t tmem_base_s;
  constexpr bool BF16 = sizeof(T) == 2 && !std::is_same<T, __half>::value;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1024-byte alignment for the swizzled tiles
  unsigned char* smem =
      smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* rot = smem;
  unsigned char* stages = smem + kRotBytes;
  constexpr uint32_t tmem_cols = 256u;
  constexpr uint32_t buf_cols = 128u;

  // ---- setup: rotation operand B[n][k] = H[n][k] D_k (+-1), barriers, TMEM
  {
    const uint16_t one = BF16 ? 0x3F80u : 0x3C00u;
    for (int e = tid; e < kDP * (kDP / 8); e += kThreads) {
      const int n = e / (kDP / 8), kc = e % (kDP / 8);
      uint16_t v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = kc * 8 + i;
        const uint32_t neg = (__popc(n & k) & 1) ^ ((qp.dmask[k >> 5] >> (k & 31)) & 1u);
        v[i] = (uint16_t)(one | (neg << 15));
      }
      uint4 w;
      w.x = v[0] | ((uint32_t)v[1] << 16);
      w.y = v[2] | ((uint32_t)v[3] << 16);
      w.z = v[4] | ((uint32_t)v[5] << 16);
      w.w = v[6] | ((uint32_t)v[7] << 16);
      *reinterpret_cast<uint4*>(rot + core_offset(n, kc * 8, kDP)) = w;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bar_accf[b]), 1);
      mbar_init(smem_u32(&bar_acce[b]), 4);
    }
    mbar_init(smem_u32(&bar_done), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_s)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const int64_t G = gridDim.x;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int L = 0;; ++L) {
        const int64_t tile = blockIdx.x + (int64_t)L * G;
        if (tile >= a.n_tiles) break;
        const int s = L % kStages;
        if (L >= kStages && !mbar_wait(smem_u32(&bar_empty[s]), ((L / kStages) - 1) & 1, a.err)) break;
        const uint32_t dst = smem_u32(stages + s * kTileBytes);
        mbar_arrive_tx(smem_u32(&bar_full[s]), kTileBytes);
        tma_load_2d(dst, &xmap, 0, (int)(tile * kRows), smem_u32(&bar_full[s]));
        tma_load_2d(dst + kTileBytes / 2, &xmap, 64, (int)(tile * kRows), smem_u32(&bar_full[s]));
        issued = L + 1;
      }
      // no copy may still be landing when the CTA exits
      for (int L = issued - kStages < 0 ? 0 : issued - kStages; L < issued; ++L)
        mbar_wait(smem_u32(&bar_full[L % kStages]), (L / kStages) & 1, a.err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t fmt = BF16 ? 1u : 0u;
      const uint32_t idesc1 = (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kDP >> 3) << 17) |
                              ((uint32_t)(kRows >> 4) << 24);
      const uint32_t rot_base = smem_u32(rot);
      for (int L = 0;; ++L) {
        const int64_t tile = blockIdx.x + (int64_t)L * G;
        const bool have = tile < a.n_tiles;
        if (have) {
          const int s = L % kStages, b = L & 1;
          if (!mbar_wait(smem_u32(&bar_full[s]), (L / kStages) & 1, a.err)) break;
          if (L >= 2 && !mbar_wait(smem_u32(&bar_acce[b]), ((L >> 1) - 1) & 1, a.err)) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(stages + s * kTileBytes);
          const uint32_t d_tmem = tmem + (uint32_t)b * buf_cols;
#pragma unroll
          for (int t = 0; t < kDP / 16; ++t) {
            const uint64_t ad = desc_sw128(a_base + (uint32_t)(t >> 2) * (kTileBytes / 2) + (uint32_t)(t & 3) * 32u);
            const uint64_t bd = desc_noswz(rot_base + (uint32_t)(2 * t) * 2048u, 2048u, 128u);
            mma_ss(d_tmem, ad, bd, idesc1, t > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bar_empty[s]));
          tc_commit(smem_u32(&bar_accf[b]));
        }
        if (!have) break;
      }
      // every MMA issued above has completed before TMEM is released
      tc_commit(smem_u32(&bar_done));
      mbar_wait(smem_u32(&bar_done), 0, a.err);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2;          // 0..7
    const int grp = ew >> 2;          // TMEM buffer / tile parity
    const int quarter = warp & 3;     // TMEM lanes 32*quarter .. +31
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t ubase = tmem + (uint32_t)grp * buf_cols + lane_off;
    const TransposeCtl tctl = make_transpose_ctl(lane);
    const int half_levels = 1 << (K - 1);
    float bpos[8], cpos[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      bpos[i] = i < half_levels - 1 ? qp.boundaries[half_levels + i] : 0.f;
      cpos[i] = UNB && i < half_levels ? qp.centroids[half_levels + i] : 0.f;
    }
    for (int L = grp;; L += 2) {
      const int64_t tile = blockIdx.x + (int64_t)L * G;
      if (tile >= a.n_tiles) break;
      const uint32_t par = (uint32_t)(L >> 1) & 1u;
      if (!mbar_wait_warp(smem_u32(&bar_accf[grp]), par, a.err)) break;
      tc_fence_after();
      const int64_t row = tile * kRows + quarter * 32 + lane;
      const bool valid = row < a.n_vec;
      const bool have = tile * kRows + quarter * 32 < a.n_vec;  // any valid row in this warp
      const int64_t seg = valid ? (int64_t)fastdiv((uint32_t)row, a.seg_div) : 0;
      const int64_t pos = valid ? row - seg * a.seg_len : 0;
      const int64_t slot = seg * a.seg_cap + pos;
      // BLOCK32: the warp's 32 rows are one block of one segment (segments hold
      // a multiple of 32 vectors and tiles start at multiples of 128 rows)
      uint32_t* blk = nullptr;
      if (BLOCK) {
        const int64_t row0 = tile * kRows + quarter * 32;
        const int64_t seg0 = (int64_t)fastdiv((uint32_t)row0, a.seg_div);
        blk = a.codes + (seg0 * (a.seg_cap / 32) + (row0 - seg0 * a.seg_len) / 32) * (int64_t)(K * kDP);
      }

      // pass 1: ||u|| over the four 32-column chunks; chunks 2 and 3 stay in
      // registers for pass 2
      uint32_t ra[32], rb[32];
      float ss0 = 0.f, ss1 = 0.f, ss2 = 0.f, ss3 = 0.f;
      auto sumsq = [&](const uint32_t (&r)[32]) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float v0 = __uint_as_float(r[i]), v1 = __uint_as_float(r[i + 1]);
          const float v2 = __uint_as_float(r[i + 2]), v3 = __uint_as_float(r[i + 3]);
          ss0 = fmaf(v0, v0, ss0);
          ss1 = fmaf(v1, v1, ss1);
          ss2 = fmaf(v2, v2, ss2);
          ss3 = fmaf(v3, v3, ss3);
        }
      };
      tmem_ld32(ubase, ra);
      tmem_ld32(ubase + 32u, rb);
      tmem_ld_wait2(ra, rb);
      sumsq(ra);
      sumsq(rb);
      tmem_ld32(ubase + 64u, ra);
      tmem_ld32(ubase + 96u, rb);
      tmem_ld_wait2(ra, rb);
      sumsq(ra);
      sumsq(rb);
      const float ssum = (ss0 + ss1) + (ss2 + ss3);       // ||u||^2 = d_pad ||x||^2
      const float nu = ssum > 0.f ? ssum * rsqrtf(ssum) : 0.f;
      if (!UNB && valid) a.norms[slot] = nu * qp.inv_sqrt_dpad;
      float th[8];
      float dot = 0.f;  // UNB: sum |u| |C[idx]| = nu <y, C[idx]>
#pragma unroll
      for (int i = 0; i < 8; ++i) th[i] = bpos[i] * nu;
      uint32_t rowq[K][4];

      // quantize chunk c (coordinates 32c .. 32c+31) held in r
      auto process = [&](const int c, const uint32_t (&r)[32]) {
        uint32_t planes[K];
        quant32_mse<K, UNB>(r, th, planes, cpos, dot);
        if (BLOCK) {
#pragma unroll
          for (int p = 0; p < K; ++p) {
            const uint32_t word = transpose32(valid ? planes[p] : 0u, tctl);
            if (have) blk[p * kDP + 32 * c + lane] = word;
          }
        } else {
#pragma unroll
          for (int p = 0; p < K; ++p) rowq[p][c] = planes[p];
        }
      };

      // pass 2: each chunk's reload from TMEM overlaps the previous chunk's work
      process(2, ra);
      tmem_ld32(ubase, ra);
      process(3, rb);
      tmem_ld_wait1(ra);
      tmem_ld32(ubase + 32u, rb);
      process(0, ra);
      tmem_ld_wait1(rb);
      // u has been read: the buffer is free for the next tile
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_acce[grp]));
      process(1, rb);
      // EDEN: n / <y, C[idx]> = (nu / sqrt(d_pad)) nu / dot
      if (UNB && valid) a.norms[slot] = dot > 0.f ? nu * qp.inv_sqrt_dpad * nu / dot : 0.f;
      if (!BLOCK && valid) {
        uint4* dst = reinterpret_cast<uint4*>(a.codes + slot * (int64_t)(K * 4));
#pragma unroll
        for (int p = 0; p < K; ++p) dst[p] = make_uint4(rowq[p][0], rowq[p][1], rowq[p][2], rowq[p][3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols));
  }
}


// ------------------------------------------------------------------ Q_prod, one thread per vector

// Q_prod with the Q_MSE kernel's work split: two epilogue groups of four
// warps take alternate tiles (group g the tiles L = g mod 2, in TMEM buffer
// g), and thread (warp w, lane l) owns TMEM lane 32 (w % 4) + l, i.e. one
// whole vector: its norm, quantization, residual and signs need no exchange
// between threads.  Per tile a group: reads u (two 32-column chunks at a
// time for the norm, then chunk by chunk), writes 2^10 r as fp16 hi + lo over
// u, signals the MMA warp, stores
// codes and norms, then waits for z = S r and packs the signs; while it waits
// for the MMA, the other group's warps on the same sub-partitions quantize
// the next tile.  The MMA warp issues u = (H D) x of tile L, then S r of
// tile L - 1.  Every wait is bounded (error word + clean exit).
template <typename T, int K>
__global__ void __launch_bounds__(kThreads, 1)
    encode_prod_rows_kernel(const __grid_constant__ CUtensorMap xmap, QParams qp, Args a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStages], bar_empty[kStages];
  __shared__ __align__(8) uint64_t bar_accf[2], bar_aready[2], bar_zf[2], bar_done;
  __shared__ uint32_t tmem_base_s;
  constexpr bool BF16 = !std::is_same<T, __half>::value;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = qp.m;
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* rot = smem;
  unsigned char* smat = smem + kRotBytes;
  unsigned char* stages = smat + m * kDP * 2;
  constexpr uint32_t tmem_cols = 512u;

  // ---- setup: rotation operand H D (+-1), S (fp16), barriers, TMEM
  {
    const uint16_t one = BF16 ? 0x3F80u : 0x3C00u;
    for (int e = tid; e < kDP * (kDP / 8); e += kThreads) {
      const int n = e / (kDP / 8), kc = e % (kDP / 8);
      uint16_t v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = kc * 8 + i;
        const uint32_t neg = (__popc(n & k) & 1) ^ ((qp.dmask[k >> 5] >> (k & 31)) & 1u);
        v[i] = (uint16_t)(one | (neg << 15));
      }
      uint4 w;
      w.x = v[0] | ((uint32_t)v[1] << 16);
      w.y = v[2] | ((uint32_t)v[3] << 16);
      w.z = v[4] | ((uint32_t)v[5] << 16);
      w.w = v[6] | ((uint32_t)v[7] << 16);
      *reinterpret_cast<uint4*>(rot + core_offset(n, kc * 8, kDP)) = w;
    }
    for (int e = tid; e < m * (kDP / 8); e += kThreads) {
      const int row = e / (kDP / 8), kc = e % (kDP / 8);
      const uint4 w = *reinterpret_cast<const uint4*>(qp.S16 + (size_t)row * kDP + kc * 8);
      *reinterpret_cast<uint4*>(smat + core_offset(row, kc * 8, m)) = w;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bar_accf[b]), 1);
      mbar_init(smem_u32(&bar_aready[b]), 128);  // every thread of the group
      mbar_init(smem_u32(&bar_zf[b]), 1);
    }
    mbar_init(smem_u32(&bar_done), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_s)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const int64_t G = gridDim.x;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int L = 0;; ++L) {
        const int64_t tile = blockIdx.x + (int64_t)L * G;
        if (tile >= a.n_tiles) break;
        const int s = L % kStages;
        if (L >= kStages && !mbar_wait(smem_u32(&bar_empty[s]), ((L / kStages) - 1) & 1, a.err)) break;
        const uint32_t dst = smem_u32(stages + s * kTileBytes);
        mbar_arrive_tx(smem_u32(&bar_full[s]), kTileBytes);
        tma_load_2d(dst, &xmap, 0, (int)(tile * kRows), smem_u32(&bar_full[s]));
        tma_load_2d(dst + kTileBytes / 2, &xmap, 64, (int)(tile * kRows), smem_u32(&bar_full[s]));
        issued = L + 1;
      }
      for (int L = issued - kStages < 0 ? 0 : issued - kStages; L < issued; ++L)
        mbar_wait(smem_u32(&bar_full[L % kStages]), (L / kStages) & 1, a.err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t fmt = BF16 ? 1u : 0u;
      const uint32_t idesc1 = (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kDP >> 3) << 17) |
                              ((uint32_t)(kRows >> 4) << 24);
      const uint32_t idesc2 = (1u << 4) | ((uint32_t)(m >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
      const uint32_t rot_base = smem_u32(rot);
      const uint32_t s_base = smem_u32(smat);
      const uint32_t s_lbo = (uint32_t)(m / 8) * 128u;
      for (int L = 0;; ++L) {
        const int64_t tile = blockIdx.x + (int64_t)L * G;
        const bool have = tile < a.n_tiles;
        if (have) {
          // u of tile L into buffer L & 1; the residual of tile L - 2 that it
          // overwrites was read by the S r MMA issued before this one
          const int s = L % kStages, b = L & 1;
          if (!mbar_wait(smem_u32(&bar_full[s]), (L / kStages) & 1, a.err)) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(stages + s * kTileBytes);
          const uint32_t d_tmem = tmem + (uint32_t)b * 256u;
#pragma unroll
          for (int t = 0; t < kDP / 16; ++t) {
            const uint64_t ad = desc_sw128(a_base + (uint32_t)(t >> 2) * (kTileBytes / 2) + (uint32_t)(t & 3) * 32u);
            const uint64_t bd = desc_noswz(rot_base + (uint32_t)(2 * t) * 2048u, 2048u, 128u);
            mma_ss(d_tmem, ad, bd, idesc1, t > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bar_empty[s]));
          tc_commit(smem_u32(&bar_accf[b]));
        }
        if (L >= 1) {
          // z = S r of tile L - 1 once its group has written the residual (the
          // group read the previous z of this buffer before that)
          const int Lp = L - 1, b = Lp & 1;
          if (!mbar_wait(smem_u32(&bar_aready[b]), (Lp >> 1) & 1, a.err)) break;
          tc_fence_after();
          const uint32_t a_tmem = tmem + (uint32_t)b * 256u;
          const uint32_t z_tmem = a_tmem + 128u;
#pragma unroll
          for (int pass = 0; pass < 2; ++pass) {  // hi, then lo parts of r
#pragma unroll
            for (int t = 0; t < kDP / 16; ++t) {
              const uint32_t acol = (uint32_t)(32 * (t >> 1) + 16 * pass + 8 * (t & 1));
              const uint64_t bd = desc_noswz(s_base + (uint32_t)(2 * t) * s_lbo, s_lbo, 128u);
              mma_ts(z_tmem, a_tmem + acol, bd, idesc2, (pass | t) ? 1u : 0u);
            }
          }
          tc_commit(smem_u32(&bar_zf[b]));
        }
        if (!have) break;
      }
      tc_commit(smem_u32(&bar_done));
      mbar_wait(smem_u32(&bar_done), 0, a.err);
    }
  } else {
    // ---------------------------------------------------------------- epilogue groups
    const int grp = (warp - 2) >> 2;  // 0 or 1: tiles L = grp mod 2, TMEM buffer grp
    const int quarter = warp & 3;     // TMEM lanes 32*quarter .. +31
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t ubase = tmem + (uint32_t)grp * 256u + lane_off;
    const int half_levels = 1 << (K - 1);
    float tc[4], dc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) tc[j] = dc[j] = 0.f;
    const float c0s = 1024.0f * qp.centroids[half_levels];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      if (j < half_levels - 1) {
        tc[j] = 1024.0f * qp.boundaries[half_levels + j] - c0s;
        dc[j] = 1024.0f * (qp.centroids[half_levels + j + 1] - qp.centroids[half_levels + j]);
      }
    }
    const int sw_words = m / 32;  // sign words per vector (2 or 4)
    for (int L = grp;; L += 2) {
      const int64_t tile = blockIdx.x + (int64_t)L * G;
      if (tile >= a.n_tiles) break;
      const uint32_t par = (uint32_t)(L >> 1) & 1u;
      if (!mbar_wait_warp(smem_u32(&bar_accf[grp]), par, a.err)) break;
      tc_fence_after();
      const int64_t row = tile * kRows + quarter * 32 + lane;
      const bool valid = row < a.n_vec;
      const int64_t seg = valid ? (int64_t)fastdiv((uint32_t)row, a.seg_div) : 0;
      const int64_t slot = seg * a.seg_cap + (valid ? row - seg * a.seg_len : 0);

      // pass 1: ||u|| over the four chunks
      uint32_t ra[32], rb[32];
      uint64_t s2a = 0, s2b = 0;
      auto sumsq = [&](const uint32_t (&r)[32]) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const uint64_t p0 = pk2(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
          const uint64_t p1 = pk2(__uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
          s2a = fma2(p0, p0, s2a);
          s2b = fma2(p1, p1, s2b);
        }
      };
      tmem_ld32(ubase, ra);
      tmem_ld32(ubase + 32u, rb);
      tmem_ld_wait2(ra, rb);
      sumsq(ra);
      sumsq(rb);
      tmem_ld32(ubase + 64u, ra);
      tmem_ld32(ubase + 96u, rb);
      tmem_ld_wait2(ra, rb);
      sumsq(ra);
      sumsq(rb);
      const float2 fa = upk2(s2a), fb = upk2(s2b);
      const float ss = (fa.x + fa.y) + (fb.x + fb.y);  // ||u||^2 = d_pad ||x||^2
      const bool zero = !(ss > 0.f);
      const float rs = rsqrtf(ss);
      const float nu = zero ? 0.f : ss * rs;
      const float inv = zero ? 0.f : 1024.0f * rs;

      // pass 2: quantize chunk c, write 2^10 r as fp16 hi (columns 32c .. 32c+15)
      // and lo (32c+16 .. 32c+31) over u
      uint64_t rr2 = 0;
      uint32_t* dst = a.codes + slot * (int64_t)(K * 4);
      auto process = [&](const int c, uint32_t (&r)[32]) {
        float (&v)[32] = *reinterpret_cast<float(*)[32]>(&r);  // quantized in place
        uint32_t NS = 0, T0 = 0, T1 = 0, T2 = 0;
        quant32_prod_sb<K>(v, tc, dc, c0s, inv, NS, T0, T1, T2);
        if (valid) {  // word c of every plane
          const uint32_t S = zero ? 0u : ~NS;
          const uint32_t M0 = K == 3 ? (T0 ^ T1 ^ T2) : T0;
          uint32_t planes[K];
          planes_from<K>(S, M0, T1, 0u, planes);
#pragma unroll
          for (int p = 0; p < K; ++p) dst[4 * p + c] = planes[p];
        }
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint32_t hiw[8], low[8];
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) {
            const float r0 = v[16 * g + 2 * qq], r1 = v[16 * g + 2 * qq + 1];
            const float h0 = __uint_as_float(__float_as_uint(r0) & 0xFFFFE000u);
            const float h1 = __uint_as_float(__float_as_uint(r1) & 0xFFFFE000u);
            const uint64_t rp = pk2(r0, r1);
            rr2 = fma2(rp, rp, rr2);
            const float2 lo = upk2(sub2(rp, pk2(h0, h1)));
            const __half2 hv = __floats2half2_rn(h0, h1);
            const __half2 lv = __floats2half2_rn(lo.x, lo.y);
            hiw[qq] = *reinterpret_cast<const uint32_t*>(&hv);
            low[qq] = *reinterpret_cast<const uint32_t*>(&lv);
          }
          tmem_st8(ubase + (uint32_t)(32 * c + 8 * g), hiw);
          tmem_st8(ubase + (uint32_t)(32 * c + 16 + 8 * g), low);
        }
      };
      // every chunk reloaded (a chunk's columns are rewritten only after it
      // has been loaded); the other group's warps cover the load latency
#pragma unroll 2
      for (int c = 0; c < 4; ++c) {
        tmem_ld32_sync(ubase + (uint32_t)(32 * c), ra);
        process(c, ra);
      }
      const float2 rrf = upk2(rr2);
      const float rr = rrf.x + rrf.y;
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_aready[grp]));
      if (valid) {
        a.norms[slot] = nu * qp.inv_sqrt_dpad;
        put_rnorm(a.rnorms, slot, rr > 0.f ? rr * rsqrtf(rr) * (1.0f / 1024.0f) : 0.f, qp.rnorm_f16);
      }
      // signs of this tile once z = S r is in TMEM (the other group's warps
      // keep the sub-partitions busy meanwhile)
      if (!mbar_wait_warp(smem_u32(&bar_zf[grp]), par, a.err)) break;
      tc_fence_after();
      for (int c = 0; c < sw_words; ++c) {
        uint32_t z[32];
        tmem_ld32_sync(tmem + (uint32_t)grp * 256u + 128u + (uint32_t)(32 * c) + lane_off, z);
        uint32_t neg = 0;
#pragma unroll
        for (int i = 31; i >= 0; --i) neg = shift_in(neg, z[i]);
        // bit i = [(S r)_(32c+i) >= 0]; a zero vector's residual was formed
        // with the opposite sign (see quant32_prod_sb)
        if (valid) a.signs[slot * sw_words + c] = zero ? neg : ~neg;
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols));
  }
}

}  // namespace enc3
}  // namespace tq
