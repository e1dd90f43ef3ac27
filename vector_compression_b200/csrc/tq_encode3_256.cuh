// Q_MSE encode with the rotation on the tensor cores at d_pad = 256 (fp16 or
// bf16 input, randomized Hadamard rotation; the method as in tq_encode3.cuh:
// TurboQuant blog notes, Q_MSE; explainer §6).
//
// The 256-point Hadamard matrix is [[H, H], [H, -H]] with H the 128-point one,
// so with x = [x1 | x2] and the sign flips D = [D1 | D2],
//   u = H256 D x = [P + Q | P - Q],  P = (H D1) x1,  Q = (H D2) x2.
// Per tile of 128 vectors the MMA warp forms P and Q (eight K = 16 MMAs each,
// M = N = 128, exact +-1 products and fp32 sums in TMEM) and the epilogue
// forms the halves of u with one addition per coordinate, then quantizes
// like the 128-point kernel: n = ||u|| / 16, the sign plane and the
// thermometer planes of |u| against the positive boundaries times ||u||.
// Shared memory: the operands H D1 and H D2 (32 KB each, no swizzle) and two
// 64 KB input stages (four 128-byte-swizzled boxes of 64 columns; columns
// d .. 255 read as zero).  Two epilogue groups of four warps take alternate
// tiles in TMEM buffers of 256 columns.  Every wait is bounded.
#pragma once

#include "tq_encode3.cuh"

namespace tq {
namespace enc3 {

constexpr int kDP2 = 256;
constexpr int kStages2 = 2;
constexpr uint32_t kTileBytes2 = kRows * kDP2 * 2;     // 64 KB: four boxes of 128 x 64
constexpr uint32_t kHalfOpBytes = kDP * kDP * 2;      // 32 KB: H D1 or H D2
inline uint32_t smem_bytes_256() { return 2 * kHalfOpBytes + kStages2 * kTileBytes2 + 1024; }

template <typename T, int K, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    encode_tc256_kernel(const __grid_constant__ CUtensorMap xmap, QParams qp, Args a) {
  constexpr bool BLOCK = MODE == MODE_MSE_BLOCK || MODE == MODE_MSE_BLOCK_U;
  constexpr bool UNB = MODE == MODE_MSE_ROW_U || MODE == MODE_MSE_BLOCK_U;  // EDEN scale
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStages2], bar_empty[kStages2];
  __shared__ __align__(8) uint64_t bar_accf[2], bar_acce[2], bar_done;
  __shared__ uint32_t tmem_base_s;
  constexpr bool BF16 = sizeof(T) == 2 && !std::is_same<T, __half>::value;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* op = smem;                        // [H D1 | H D2]
  unsigned char* stages = smem + 2 * kHalfOpBytes;
  constexpr uint32_t tmem_cols = 512u;
  constexpr uint32_t buf_cols = 256u;              // P in columns 0..127, Q in 128..255

  // ---- setup: operands B_h[n][k] = H[n][k] D_(128 h + k) (+-1), barriers, TMEM
  {
    const uint16_t one = BF16 ? 0x3F80u : 0x3C00u;
    for (int e = tid; e < 2 * kDP * (kDP / 8); e += kThreads) {
      const int h = e / (kDP * (kDP / 8)), r = e % (kDP * (kDP / 8));
      const int n = r / (kDP / 8), kc = r % (kDP / 8);
      uint16_t v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = kc * 8 + i, kd = kDP * h + k;
        const uint32_t neg = (__popc(n & k) & 1) ^ ((qp.dmask[kd >> 5] >> (kd & 31)) & 1u);
        v[i] = (uint16_t)(one | (neg << 15));
      }
      uint4 w;
      w.x = v[0] | ((uint32_t)v[1] << 16);
      w.y = v[2] | ((uint32_t)v[3] << 16);
      w.z = v[4] | ((uint32_t)v[5] << 16);
      w.w = v[6] | ((uint32_t)v[7] << 16);
      *reinterpret_cast<uint4*>(op + h * kHalfOpBytes + core_offset(n, kc * 8, kDP)) = w;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kStages2; ++s) {
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
        const int s = L % kStages2;
        if (L >= kStages2 && !mbar_wait(smem_u32(&bar_empty[s]), ((L / kStages2) - 1) & 1, a.err)) break;
        const uint32_t dst = smem_u32(stages + s * kTileBytes2);
        mbar_arrive_tx(smem_u32(&bar_full[s]), kTileBytes2);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_load_2d(dst + (uint32_t)bx * (kTileBytes2 / 4), &xmap, 64 * bx, (int)(tile * kRows),
                      smem_u32(&bar_full[s]));
        issued = L + 1;
      }
      // no copy may still be landing when the CTA exits
      for (int L = issued - kStages2 < 0 ? 0 : issued - kStages2; L < issued; ++L)
        mbar_wait(smem_u32(&bar_full[L % kStages2]), (L / kStages2) & 1, a.err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t fmt = BF16 ? 1u : 0u;
      const uint32_t idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kDP >> 3) << 17) |
                             ((uint32_t)(kRows >> 4) << 24);
      const uint32_t op_base = smem_u32(op);
      for (int L = 0;; ++L) {
        const int64_t tile = blockIdx.x + (int64_t)L * G;
        if (tile >= a.n_tiles) break;
        const int s = L % kStages2, b = L & 1;
        if (!mbar_wait(smem_u32(&bar_full[s]), (L / kStages2) & 1, a.err)) break;
        if (L >= 2 && !mbar_wait(smem_u32(&bar_acce[b]), ((L >> 1) - 1) & 1, a.err)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(stages + s * kTileBytes2);
        // P = x1 (H D1)^T into columns 0..127, Q = x2 (H D2)^T into 128..255
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t d_tmem = tmem + (uint32_t)b * buf_cols + (uint32_t)h * kDP;
#pragma unroll
          for (int t = 0; t < kDP / 16; ++t) {
            const int box = 2 * h + (t >> 2);
            const uint64_t ad = desc_sw128(a_base + (uint32_t)box * (kTileBytes2 / 4) + (uint32_t)(t & 3) * 32u);
            const uint64_t bd = desc_noswz(op_base + (uint32_t)h * kHalfOpBytes + (uint32_t)(2 * t) * 2048u, 2048u, 128u);
            mma_ss(d_tmem, ad, bd, idesc, t > 0 ? 1u : 0u);
          }
        }
        tc_commit(smem_u32(&bar_empty[s]));
        tc_commit(smem_u32(&bar_accf[b]));
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
    const uint32_t pbase = tmem + (uint32_t)grp * buf_cols + lane_off;  // P; Q 128 columns on
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
        blk = a.codes + (seg0 * (a.seg_cap / 32) + (row0 - seg0 * a.seg_len) / 32) * (int64_t)(K * kDP2);
      }

      // coordinates 32 j + i of u into rp (P + Q) and 128 + 32 j + i into rq (P - Q)
      uint32_t rp[32], rq[32];
      auto load_u = [&](int j) {
        tmem_ld32(pbase + 32u * (uint32_t)j, rp);
        tmem_ld32(pbase + (uint32_t)kDP + 32u * (uint32_t)j, rq);
        tmem_ld_wait2(rp, rq);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = __uint_as_float(rp[i]), q = __uint_as_float(rq[i]);
          rp[i] = __float_as_uint(p + q);
          rq[i] = __float_as_uint(p - q);
        }
      };
      // pass 1: ||u||^2 over the 256 coordinates
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
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        load_u(j);
        sumsq(rp);
        sumsq(rq);
      }
      const float ssum = (ss0 + ss1) + (ss2 + ss3);  // ||u||^2 = d_pad ||x||^2
      const float nu = ssum > 0.f ? ssum * rsqrtf(ssum) : 0.f;
      if (!UNB && valid) a.norms[slot] = nu * qp.inv_sqrt_dpad;
      float th[8];
      float dot = 0.f;  // UNB: sum |u| |C[idx]| = nu <y, C[idx]>
#pragma unroll
      for (int i = 0; i < 8; ++i) th[i] = bpos[i] * nu;
      uint32_t rowq[K][8];

      // quantize chunk c (coordinates 32c .. 32c+31) held in r
      auto process = [&](const int c, const uint32_t (&r)[32]) {
        uint32_t planes[K];
        quant32_mse<K, UNB>(r, th, planes, cpos, dot);
        if (BLOCK) {
#pragma unroll
          for (int p = 0; p < K; ++p) {
            const uint32_t word = transpose32(valid ? planes[p] : 0u, tctl);
            if (have) blk[p * kDP2 + 32 * c + lane] = word;
          }
        } else {
#pragma unroll
          for (int p = 0; p < K; ++p) rowq[p][c] = planes[p];
        }
      };

      // pass 2: every chunk reloaded; the buffer is released after the last load
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        load_u(j);
        if (j == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_acce[grp]));
        }
        process(j, rp);
        process(4 + j, rq);
      }
      // EDEN: n / <y, C[idx]> = (nu / sqrt(d_pad)) nu / dot
      if (UNB && valid) a.norms[slot] = dot > 0.f ? nu * qp.inv_sqrt_dpad * nu / dot : 0.f;
      if (!BLOCK && valid) {
        uint4* dst = reinterpret_cast<uint4*>(a.codes + slot * (int64_t)(K * 8));
#pragma unroll
        for (int p = 0; p < K; ++p) {
          dst[2 * p] = make_uint4(rowq[p][0], rowq[p][1], rowq[p][2], rowq[p][3]);
          dst[2 * p + 1] = make_uint4(rowq[p][4], rowq[p][5], rowq[p][6], rowq[p][7]);
        }
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

}  // namespace enc3
}  // namespace tq
