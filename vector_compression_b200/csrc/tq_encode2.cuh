// Encode kernels, thread-per-vector form (d_pad = 128 or 256).
//
// Same method as tq_encode.cuh (TurboQuant blog notes, Q_MSE and the
// definition of Q_prod; explainer §6, §8): n = ||x||, y = H D x / (sqrt(d_pad) n),
// idx = #{k : B_k < y}, bit-packed codes; Q_prod adds r = y - C[idx],
// rho = ||r|| and the sign bits of S r.
//
// Work split: one warp owns a block of 32 consecutive vectors of a segment
// and one thread owns one vector, so every per-coordinate step is a single
// warp instruction for 32 vectors:
//   * rows are staged into padded shared memory with cp.async (coalesced
//     16-byte copies, double-buffered per warp);
//   * the randomized Hadamard transform runs in 128 registers per thread,
//     on packed f32x2 pairs {v_i, v_(i+64)} for the six stages that pair
//     registers across pairs;
//   * quantization uses the odd symmetry of the Lloyd-Max codebook: the sign
//     plane is [y > 0] and the magnitude index is a binary search of |y|
//     against the positive boundaries, all compared in the unscaled domain
//     (thresholds B n sqrt(d_pad));  the bit planes are shifted into
//     per-thread words (bit i = coordinate 32w + i);
//   * the BLOCK32 value layout (bit t = vector t) is produced by a 32x32
//     bit transpose across the warp (5 shuffle rounds);
//   * Q_prod: each thread writes its residual, split into fp16 hi + lo parts
//     (scaled by a power of two), into its own TMEM lane; one thread issues
//     tcgen05 MMAs D = A_hi S^T + A_lo S^T (M = 128 vectors of the CTA,
//     N = m, K = d_pad) with S resident in shared memory, and every thread
//     reads its row of D back to form the QJL sign words.
// Exact boundary ties on the negative side resolve toward zero here (the
// oracle resolves them to the lower cell); such values lie inside the
// parity window by definition.
#pragma once

#include "tq_device.cuh"
#include "tq_wait.cuh"

namespace tq {
namespace enc2 {

constexpr int kThreads = 128;

// ------------------------------------------------------------------ packed fp32 pairs

__device__ __forceinline__ uint64_t pk(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float lo_of(uint64_t r) {
  return __uint_as_float((uint32_t)(r & 0xFFFFFFFFull));
}
__device__ __forceinline__ float hi_of(uint64_t r) { return __uint_as_float((uint32_t)(r >> 32)); }
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
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

// Unnormalized 128-point Walsh-Hadamard transform of v[0..128) held as
// P[i] = {v_i, v_(i+64)}: stages h = 1..32 on packed pairs, stage 64 inside
// each pair.  Returns the result in the same packing.
__device__ __forceinline__ void fwht128(uint64_t (&P)[64]) {
#pragma unroll
  for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if ((i & h) == 0) {
        const uint64_t a = P[i], b = P[i + h];
        P[i] = add2(a, b);
        P[i + h] = sub2(a, b);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float a = lo_of(P[i]), b = hi_of(P[i]);
    P[i] = pk(a + b, a - b);
  }
}

// ------------------------------------------------------------------ staging

struct Stage {
  const unsigned char* x;  // input base (bytes)
  int64_t ld_bytes;        // row stride in bytes
  int row_bytes;           // bytes of one input row (d * esz), a multiple of 16
  int pitch;               // staged row pitch in bytes (odd number of 16-byte chunks)
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The warp copies rows [row0, row0 + nv) into buf (row r at r * pitch).
__device__ __forceinline__ void stage_rows(const Stage& st, unsigned char* buf, int64_t row0, int nv,
                                           int lane) {
  const int cpr = st.row_bytes >> 4;
  const int total = 32 * cpr;
  for (int q = lane; q < total; q += 32) {
    const int r = q / cpr, c = q - r * cpr;
    if (r < nv)
      cp_async16(buf + r * st.pitch + c * 16, st.x + (row0 + r) * st.ld_bytes + (int64_t)c * 16);
  }
}

// Sign flips of D, as XOR masks: for 16-bit inputs one word per coordinate
// pair (bits 15 and 31), for fp32 one word per coordinate (bit 31).
struct SignMasks {
  uint32_t m[kMaxHadamard];
};

// Load 8 consecutive coordinates [8c, 8c + 8) of the staged row (c < row_bytes/16 for
// 16-bit types; fp32 uses two chunks) with D applied, as floats.
// `chunks` = 16-byte chunks in the row; an fp32 row whose length is 4 mod 8
// ends with half of an 8-coordinate group, whose upper half reads as zeros.
template <typename T>
__device__ __forceinline__ void load8(const unsigned char* row, int c, const SignMasks& sg, float (&o)[8],
                                      int chunks);

template <>
__device__ __forceinline__ void load8<__half>(const unsigned char* row, int c, const SignMasks& sg,
                                              float (&o)[8], int) {
  uint4 w = *reinterpret_cast<const uint4*>(row + c * 16);
  w.x ^= sg.m[4 * c + 0];
  w.y ^= sg.m[4 * c + 1];
  w.z ^= sg.m[4 * c + 2];
  w.w ^= sg.m[4 * c + 3];
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const unsigned char* row, int c,
                                                     const SignMasks& sg, float (&o)[8], int) {
  uint4 w = *reinterpret_cast<const uint4*>(row + c * 16);
  w.x ^= sg.m[4 * c + 0];
  w.y ^= sg.m[4 * c + 1];
  w.z ^= sg.m[4 * c + 2];
  w.w ^= sg.m[4 * c + 3];
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(ws[i] << 16);
    o[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<float>(const unsigned char* row, int c, const SignMasks& sg,
                                             float (&o)[8], int chunks) {
  const uint4 a = *reinterpret_cast<const uint4*>(row + c * 32);
  const bool full = 2 * c + 1 < chunks;
  const uint4 b = full ? *reinterpret_cast<const uint4*>(row + c * 32 + 16) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t ws[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = __uint_as_float(ws[i] ^ (i < 4 || full ? sg.m[8 * c + i] : 0u));
}

// ------------------------------------------------------------------ quantize + pack

// Thresholds for one vector: positive boundaries times sigma = n sqrt(d_pad),
// and the positive centroids (for the residual).
template <int K>
struct Thr {
  float t[(1 << (K - 1)) > 1 ? (1 << (K - 1)) - 1 : 1];
};

// Quantize 32 coordinates v[0..32) (coordinate 32w + i in v[i]) and shift
// the bit planes into words (bit i = coordinate 32w + i): the sign plane
// S = [y > 0] and the magnitude bits of the binary search over the positive
// thresholds; the planes of idx = s ? 2^(K-1) + mu : 2^(K-1) - 1 - mu are
// then the top plane S and lower planes ~(S ^ M).  With RESID, v[i] is
// replaced by the residual r = v * scale - C[idx] and rr accumulates r^2.
// With DOT, dot accumulates |v| |C[idx]| (= <v, C[idx]>, same signs).
template <int K, bool RESID, bool DOT = false>
__device__ __forceinline__ void quant32(float (&v)[32], const Thr<K>& th, const float (&cpos)[8],
                                        float scale, uint32_t (&plane)[K], float& rr, float& dot) {
  uint32_t S = 0, M0 = 0, M1 = 0, M2 = 0;
#pragma unroll
  for (int i = 31; i >= 0; --i) {
    const float y = v[i];
    const float a = fabsf(y);
    const bool s = y > 0.0f;
    float cm = cpos[0];
    if (K == 2) {
      const bool m0 = a > th.t[0];
      M0 = (M0 << 1) | (m0 ? 1u : 0u);
      if (RESID || DOT) cm = m0 ? cpos[1] : cpos[0];
    } else if (K == 3) {
      const bool m1 = a > th.t[1];
      const float t0 = m1 ? th.t[2] : th.t[0];
      const bool m0 = a > t0;
      M1 = (M1 << 1) | (m1 ? 1u : 0u);
      M0 = (M0 << 1) | (m0 ? 1u : 0u);
      if (RESID || DOT) cm = m1 ? (m0 ? cpos[3] : cpos[2]) : (m0 ? cpos[1] : cpos[0]);
    } else if (K == 4) {
      const bool m2 = a > th.t[3];
      const float t1 = m2 ? th.t[5] : th.t[1];
      const bool m1 = a > t1;
      const float t0 = m1 ? (m2 ? th.t[6] : th.t[2]) : (m2 ? th.t[4] : th.t[0]);
      const bool m0 = a > t0;
      M2 = (M2 << 1) | (m2 ? 1u : 0u);
      M1 = (M1 << 1) | (m1 ? 1u : 0u);
      M0 = (M0 << 1) | (m0 ? 1u : 0u);
      if (DOT)
        cm = m2 ? (m1 ? (m0 ? cpos[7] : cpos[6]) : (m0 ? cpos[5] : cpos[4]))
                : (m1 ? (m0 ? cpos[3] : cpos[2]) : (m0 ? cpos[1] : cpos[0]));
    }
    if (DOT) dot = fmaf(a, cm, dot);
    S = (S << 1) | (s ? 1u : 0u);
    if (RESID) {
      const float r = fmaf(y, scale, s ? -cm : cm);
      v[i] = r;
      rr = fmaf(r, r, rr);
    }
  }
  plane[K - 1] = S;
  if (K >= 2) plane[0] = ~(S ^ M0);
  if (K >= 3) plane[1] = ~(S ^ M1);
  if (K >= 4) plane[2] = ~(S ^ M2);
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

// ------------------------------------------------------------------ tcgen05 helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// K-major operand tile without swizzle: 8x8 core matrices of 128 bytes,
// core (row group rg, k chunk kc) at ((kc * rows/8) + rg) * 128 bytes.
__device__ __forceinline__ uint32_t core_offset(int row, int k, int rows) {
  return (uint32_t)(((k >> 3) * (rows >> 3) + (row >> 3)) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // sm100 descriptor version; no swizzle, base offset 0
  return d;
}

__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
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

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Bounded wait for the mbarrier phase with the given parity: false, and the
// device error word set, if it does not complete within the wait budget.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* err) {
  return bounded_wait<true>(bar, parity, err);
}

// ------------------------------------------------------------------ kernel

// *_U: Q_MSE with the unbiased (EDEN) scale n / <y, C[idx]> stored as the norm
enum { MODE_MSE_ROW = 0, MODE_MSE_BLOCK = 1, MODE_PROD = 2, MODE_MSE_ROW_U = 3, MODE_MSE_BLOCK_U = 4 };

struct Args {
  Stage st;
  int64_t seg_len, seg_cap, bps, n_tasks;
  uint32_t* codes;
  uint32_t* signs;
  float* norms;
  float* rnorms;
  int nbuf;
  int tmem_cols;  // PROD: allocated TMEM columns
  unsigned* err;  // device error word (bounded-wait expiry)
};

// Dynamic shared memory: [S tile (PROD) | staging buffers (4 warps x nbuf x 32 rows)].
template <int DP, typename T, int K, int MODE>
__global__ void __launch_bounds__(kThreads, 1) encode_kernel(QParams qp, SignMasks sg, Args a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t mbar;
  __shared__ uint32_t tmem_base_s;
  constexpr bool PROD = MODE == MODE_PROD;
  constexpr bool BLOCK = MODE == MODE_MSE_BLOCK || MODE == MODE_MSE_BLOCK_U;
  constexpr bool UNB = MODE == MODE_MSE_ROW_U || MODE == MODE_MSE_BLOCK_U;
  constexpr int HALVES = DP / 128;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = qp.m;
  const int s_bytes = PROD ? m * DP * 2 : 0;
  unsigned char* stage_base = smem + s_bytes + warp * a.nbuf * 32 * a.st.pitch;

  uint32_t tmem = 0;
  if (PROD) {
    // S (fp16) into the K-major core-matrix layout: rows = m (N), K = DP.
    for (int e = tid; e < m * (DP / 8); e += kThreads) {
      const int row = e / (DP / 8), kc = e % (DP / 8);
      const uint4 w = *reinterpret_cast<const uint4*>(qp.S16 + (size_t)row * DP + kc * 8);
      *reinterpret_cast<uint4*>(smem + core_offset(row, kc * 8, m)) = w;
    }
    if (tid == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&mbar)));
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&tmem_base_s)),
                   "r"(a.tmem_cols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem = tmem_base_s;
  }

  const TransposeCtl tctl = make_transpose_ctl(lane);
  const int half_levels = 1 << (K - 1);
  // positive boundaries (B_{2^(K-1)} .. B_{2^K - 2}) and positive centroids
  float bpos[7], cpos[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) bpos[i] = i < half_levels - 1 ? qp.boundaries[half_levels + i] : 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) cpos[i] = i < half_levels ? qp.centroids[half_levels + i] : 0.f;

  const int64_t step = (int64_t)gridDim.x * 4;
  int64_t base = (int64_t)blockIdx.x * 4;
  uint32_t phase = 0;
  int cur = 0;
  // prefetch the first task
  if (a.nbuf == 2 && base + warp < a.n_tasks) {
    const int64_t task = base + warp;
    const int64_t s = task / a.bps, b = task % a.bps;
    const int nv = (int)min64(32, a.seg_len - 32 * b);
    stage_rows(a.st, stage_base, s * a.seg_len + 32 * b, nv, lane);
  }
  if (a.nbuf == 2) cp_async_commit();

  for (; base < a.n_tasks; base += step) {
    const int64_t task = base + warp;
    const bool have = task < a.n_tasks;
    int64_t s = 0, b = 0;
    int nv = 0;
    if (have) {
      s = task / a.bps;
      b = task % a.bps;
      nv = (int)min64(32, a.seg_len - 32 * b);
    }
    unsigned char* buf = stage_base + cur * 32 * a.st.pitch;
    if (a.nbuf == 2) {
      const int64_t nt = task + step;
      if (nt < a.n_tasks) {
        const int64_t ns = nt / a.bps, nbk = nt % a.bps;
        const int nnv = (int)min64(32, a.seg_len - 32 * nbk);
        stage_rows(a.st, stage_base + (cur ^ 1) * 32 * a.st.pitch, ns * a.seg_len + 32 * nbk, nnv, lane);
      }
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      if (have) stage_rows(a.st, buf, s * a.seg_len + 32 * b, nv, lane);
      cp_async_commit();
      cp_async_wait<0>();
    }
    __syncwarp();

    const bool valid = have && lane < nv;
    uint32_t rowq[K][4];
    const unsigned char* row = buf + lane * a.st.pitch;
    const int64_t slot = s * a.seg_cap + 32 * b + lane;
    const int chunks = a.st.row_bytes >> 4;  // 16-byte chunks of the input row
    constexpr int ESZ = sizeof(T);

    // ---- per half (DP = 256: y_lo = H(x_lo + x_hi), y_hi = H(x_lo - x_hi))
    float nrm2 = 0.f, rr2 = 0.f, scale = 0.f, nrm = 0.f, dot = 0.f;
    Thr<K> th;
#pragma unroll
    for (int i = 0; i < (int)(sizeof(th.t) / sizeof(float)); ++i) th.t[i] = 0.f;
#pragma unroll 1
    for (int hf = 0; hf < HALVES; ++hf) {
      uint64_t P[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {  // coordinates [8c, 8c + 8) of the half
        float lo8[8], hi8[8];
        const bool in_lo = ESZ == 2 ? (c < chunks) : (2 * c < chunks);
        const bool in_hi = HALVES == 2 && (ESZ == 2 ? (c + 16 < chunks) : (2 * (c + 16) < chunks));
        if (in_lo) load8<T>(row, c, sg, lo8, chunks);
        else {
#pragma unroll
          for (int i = 0; i < 8; ++i) lo8[i] = 0.f;
        }
        if (in_hi) load8<T>(row, c + 16, sg, hi8, chunks);
        else {
#pragma unroll
          for (int i = 0; i < 8; ++i) hi8[i] = 0.f;
        }
        if (hf == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) nrm2 = fmaf(lo8[i], lo8[i], fmaf(hi8[i], hi8[i], nrm2));
        }
        // pack coordinates j = 8c + i as P[j mod 64] = {v_j, v_(j+64)}
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 8 * c + i;
          const float val = HALVES == 1 ? lo8[i] : (hf == 0 ? lo8[i] + hi8[i] : lo8[i] - hi8[i]);
          if (j < 64) P[j] = pk(val, 0.f);
          else P[j - 64] = pk(lo_of(P[j - 64]), val);
        }
      }
      if (hf == 0) {
        const float n = sqrtf(nrm2);
        const float sigma = n * sqrtf((float)DP);
        scale = n > 0.f ? qp.inv_sqrt_dpad / n : 0.f;
        nrm = n;
#pragma unroll
        for (int i = 0; i < (int)(sizeof(th.t) / sizeof(float)); ++i) th.t[i] = bpos[i] * sigma;
        if (!UNB && valid) a.norms[slot] = n;
      }
      fwht128(P);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = 32 * w + i;
          v[i] = j < 64 ? lo_of(P[j]) : hi_of(P[j - 64]);
        }
        uint32_t planes[K];
        quant32<K, PROD, UNB>(v, th, cpos, scale, planes, rr2, dot);
        if (BLOCK) {
          uint32_t* dst = a.codes + (s * (a.seg_cap / 32) + b) * (int64_t)(K * DP);
#pragma unroll
          for (int p = 0; p < K; ++p) {
            const uint32_t word = transpose32(valid ? planes[p] : 0u, tctl);
            if (have) dst[p * DP + 128 * hf + 32 * w + lane] = word;
          }
        } else {
#pragma unroll
          for (int p = 0; p < K; ++p) rowq[p][w] = planes[p];
        }
        if (PROD) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int j = 32 * w + i;
            if (j < 64) P[j] = pk(v[i], hi_of(P[j]));
            else P[j - 64] = pk(lo_of(P[j - 64]), v[i]);
          }
        }
      }
      if (!BLOCK && valid) {
        uint32_t* dst = a.codes + slot * (int64_t)(K * DP / 32);
#pragma unroll
        for (int p = 0; p < K; ++p)
          *reinterpret_cast<uint4*>(dst + p * (DP / 32) + 4 * hf) =
              make_uint4(rowq[p][0], rowq[p][1], rowq[p][2], rowq[p][3]);
      }
      if (PROD) {
        // stash this half's residual in TMEM as fp16 hi and lo parts
        // (A_hi at columns [0, DP/2), A_lo at [DP/2, DP)).  r is a difference
        // of unit-vector coordinates, |r_j| <= 1, so the exact scale 2^10 keeps
        // the hi part below the fp16 maximum and the lo part out of the
        // subnormal range; the sign of S r is unchanged by the scale.
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {  // 16 columns = 32 coordinates
          uint32_t hiw[16], low[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int j = 2 * (c0 + q);
            const float r0 = 1024.0f * (j < 64 ? lo_of(P[j]) : hi_of(P[j - 64]));
            const float r1 = 1024.0f * ((j + 1) < 64 ? lo_of(P[j + 1]) : hi_of(P[j + 1 - 64]));
            const __half2 h = __floats2half2_rn(r0, r1);
            const float2 hf2 = __half22float2(h);
            const __half2 l = __floats2half2_rn(r0 - hf2.x, r1 - hf2.y);
            hiw[q] = *reinterpret_cast<const uint32_t*>(&h);
            low[q] = *reinterpret_cast<const uint32_t*>(&l);
          }
          const uint32_t col = (uint32_t)(hf * 64 + c0);
          tmem_st16(lane_base + col, hiw);
          tmem_st16(lane_base + (uint32_t)(DP / 2) + col, low);
        }
      }
    }

    if (UNB && valid) {  // EDEN's scale n / <y, C[idx]>, with <y, C[idx]> = scale * dot
      const float yc = dot * scale;
      a.norms[slot] = yc > 0.f ? nrm / yc : 0.f;
    }
    if (PROD) {
      const float rho = sqrtf(rr2);
      if (valid) put_rnorm(a.rnorms, slot, rho, qp.rnorm_f16);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        // D[128 x m] = A_hi S^T + A_lo S^T, K = DP in steps of 16
        const uint32_t idesc = (1u << 4) | ((uint32_t)(m >> 3) << 17) | ((128u >> 4) << 24);
        const uint32_t lbo = (uint32_t)(m / 8) * 128u;
        const uint32_t d_tmem = tmem + (uint32_t)DP;  // D after A_hi, A_lo
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
          for (int ks = 0; ks < DP / 16; ++ks) {
            const uint64_t bdesc = smem_desc(smem_u32(smem) + (uint32_t)(2 * ks) * lbo, lbo, 128u);
            const uint32_t a_tmem = tmem + (uint32_t)(pass * (DP / 2) + ks * 8);
            const uint32_t acc = (pass | ks) ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
                "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc));
          }
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&mbar))
            : "memory");
      }
      // the decision to continue must be the same for every thread of the CTA
      const bool ok = __syncthreads_and(mbar_wait(smem_u32(&mbar), phase, a.err) ? 1 : 0) != 0;
      phase ^= 1u;
      tc_fence_after();
      if (!ok) break;  // bounded wait expired: error word set, stop this CTA
      {
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)DP;
        for (int c0 = 0; c0 < m; c0 += 32) {
          uint32_t z[32];
          tmem_ld32(lane_base + (uint32_t)c0, z);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          uint32_t word = 0;
#pragma unroll
          for (int i = 31; i >= 0; --i) word = (word << 1) | (__uint_as_float(z[i]) >= 0.0f ? 1u : 0u);
          if (valid) a.signs[slot * (int64_t)(m / 32) + c0 / 32] = word;
        }
      }
      tc_fence_before();
      __syncthreads();  // D and A are rewritten by the next tile
      tc_fence_after();
    }
    __syncwarp();
    cur ^= (a.nbuf == 2) ? 1 : 0;
  }
  cp_async_wait<0>();
  if (PROD) {
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(a.tmem_cols));
  }
}

}  // namespace enc2
}  // namespace tq
