// Split-precision fp32 products on the tcgen05 tensor cores (interface and
// the precision argument in tq_gemm_tc.h).
//
// A persistent CTA per SM walks the output tiles of 128 x 128 (tile t: row
// block t / (N / 128), column block t % (N / 128), so CTAs that run at the
// same time share row blocks of A in L2, and B stays in L2).  K is taken in
// chunks of 64 columns; a chunk's MMAs (every term, in the given order)
// accumulate into one of four 128-column TMEM accumulators.
//   warp 0      TMA producer: per pipeline stage the 128 x 64 boxes (128-byte
//               swizzle) of the chunk's distinct A and B column ranges, each
//               loaded once however many terms read it, in a ring of as
//               many stages as 192 KB holds (3 for four boxes, 4 for three);
//   warp 1      TMEM allocator (512 columns) and MMA issuer: tcgen05.mma
//               kind::f16 (M 128, N 128, K 16), fp32 accumulation;
//   warps 2..9  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its 32
//               rows), columns 64 h .. 64 h + 63 with h = (w - 2) / 4, adds
//               each chunk's sums into 64 fp32 registers per row (round to
//               nearest), releases the accumulator, and after the last chunk
//               stores its 64 scaled values of the row.
// Every wait is bounded (device error word + clean exit).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "tq_device.cuh"
#include "tq_gemm_tc.h"
#include "tq_wait.cuh"

namespace tq {
namespace gemm_tc {

namespace {

constexpr int kMaxStages = 6;
constexpr int kAcc = 4;  // chunk accumulators in TMEM
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxBoxes = 4;                              // distinct A + B ranges per stage
constexpr uint32_t kBoxBytes = kBM * kBK * 2;              // 16 KB (kBM == kBN)
constexpr uint32_t kRing = 192 * 1024;                     // stage ring bytes
constexpr uint32_t kSmem = kRing + 1024;
static_assert(kBM == kBN && kKC == kBK, "one box size, one stage per chunk");

struct Args {
  int64_t M;
  int N, K, nterms;
  int na, nb;                   // distinct A and B column ranges
  int a_base0, a_base1, a_base2;  // their first columns
  int b_base0, b_base1, b_base2;
  int ia0, ia1, ia2, ib0, ib1, ib2;  // term t reads A box ia_t and B box ib_t
  int stages;                        // ring stages of (na + nb) boxes
  float scale;
  float* C;
  int64_t ldc;
  int tiles_n;
  int64_t n_tiles;
  unsigned* err;
};

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
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, unsigned* err) {
  return bounded_wait<true>(bar, parity, err);
}
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, unsigned* err) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, err)) != 0;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// D (TMEM) (+)= A (smem descriptor) * B (smem descriptor)^T, fp16 in, fp32 out
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc));
}
// K-major operand written by TMA with the 128-byte swizzle: rows of 128
// bytes, 8-row groups 1024 bytes apart; the start address moves by 32 bytes
// per 16 fp16 of K inside the swizzle row.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
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
// completes this thread's outstanding tcgen05.ld; the empty statements keep
// every use of the registers after the wait
__device__ __forceinline__ void tmem_ld_wait2(uint32_t (&r)[32], uint32_t (&q)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]), "+r"(q[i]));
}

__device__ __forceinline__ int pick(int t, int v0, int v1, int v2) { return t == 0 ? v0 : (t == 1 ? v1 : v2); }

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap, Args a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kMaxStages], bar_empty[kMaxStages], bar_pfull[kAcc], bar_pempty[kAcc],
      bar_done;
  __shared__ uint32_t tmem_base_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(smem_u32(&bar_pfull[b]), 1);
      mbar_init(smem_u32(&bar_pempty[b]), kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(&bar_done), 1);
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
  const int n_chunks = a.K / kKC;  // K chunks (= pipeline stages) per tile
  const uint32_t nst = (uint32_t)a.stages, stage_bytes = (uint32_t)(a.na + a.nb) * kBoxBytes;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        const int mb = (int)(tile / a.tiles_n), nb = (int)(tile % a.tiles_n);
        for (int c = 0; c < n_chunks; ++c, ++it) {
          const uint32_t s = it % nst;
          if (it >= nst && !wait_bar(smem_u32(&bar_empty[s]), ((it / nst) - 1) & 1u, a.err)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const uint32_t bar = smem_u32(&bar_full[s]);
          mbar_expect(bar, (uint32_t)(a.na + a.nb) * kBoxBytes);
          for (int i = 0; i < a.na; ++i)
            tma_load_2d(sa + i * kBoxBytes, &amap, pick(i, a.a_base0, a.a_base1, a.a_base2) + c * kKC, mb * kBM, bar);
          for (int j = 0; j < a.nb; ++j)
            tma_load_2d(sa + (a.na + j) * kBoxBytes, &bmap, pick(j, a.b_base0, a.b_base1, a.b_base2) + c * kKC,
                        nb * kBN, bar);
        }
      }
      // the CTA leaves no copy in flight
      for (uint32_t c = it > nst ? it - nst : 0; c < it; ++c)
        wait_bar(smem_u32(&bar_full[c % nst]), (c / nst) & 1u, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = (1u << 4) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      uint32_t it = 0, gc = 0;  // stages and chunks so far
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        for (int c = 0; ok && c < n_chunks; ++c, ++gc) {
          const uint32_t pb = gc % kAcc;
          if (gc >= (uint32_t)kAcc && !wait_bar(smem_u32(&bar_pempty[pb]), ((gc / kAcc) - 1) & 1u, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + pb * (uint32_t)kBN;
          const uint32_t s = it % nst;
          if (!wait_bar(smem_u32(&bar_full[s]), (it / nst) & 1u, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          for (int t = 0; t < a.nterms; ++t) {
            const uint32_t ab = sa + (uint32_t)pick(t, a.ia0, a.ia1, a.ia2) * kBoxBytes;
            const uint32_t bb = sa + (uint32_t)(a.na + pick(t, a.ib0, a.ib1, a.ib2)) * kBoxBytes;
#pragma unroll
            for (int k4 = 0; k4 < kBK / 16; ++k4)
              mma_f16(d, desc_sw128(ab + 32u * k4), desc_sw128(bb + 32u * k4), idesc, (t | k4) ? 1u : 0u);
          }
          tc_commit(smem_u32(&bar_empty[s]));
          ++it;
          if (!ok) break;
          tc_commit(smem_u32(&bar_pfull[pb]));
        }
      }
      tc_commit(smem_u32(&bar_done));
      wait_bar(smem_u32(&bar_done), 0, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3, h = (warp - 2) >> 2;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    constexpr int kCols = kBN / 2;  // columns per thread
    uint32_t gc = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
      const int mb = (int)(tile / a.tiles_n), nb = (int)(tile % a.tiles_n);
      float acc[kCols];  // this row's sums over the chunks so far
#pragma unroll
      for (int j = 0; j < kCols; ++j) acc[j] = 0.f;
      for (int c = 0; c < n_chunks; ++c, ++gc) {
        const uint32_t pb = gc % kAcc;
        if (!wait_bar_warp(smem_u32(&bar_pfull[pb]), (gc / kAcc) & 1u, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        const uint32_t col = tmem + pb * (uint32_t)kBN + lane_off + (uint32_t)(kCols * h);
        tmem_ld32(col, r0);
        tmem_ld32(col + 32u, r1);
        tmem_ld_wait2(r0, r1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          acc[i] += __uint_as_float(r0[i]);
          acc[32 + i] += __uint_as_float(r1[i]);
        }
        // the accumulator has been read: free for the chunk kAcc later
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_pempty[pb]));
      }
      if (!ok) break;
      const int64_t row = (int64_t)mb * kBM + 32 * q + lane;
      if (row < a.M) {
        float4* dst = reinterpret_cast<float4*>(a.C + row * a.ldc + (int64_t)nb * kBN + kCols * h);
#pragma unroll
        for (int v = 0; v < kCols / 4; ++v)
          dst[v] = make_float4(a.scale * acc[4 * v], a.scale * acc[4 * v + 1], a.scale * acc[4 * v + 2],
                               a.scale * acc[4 * v + 3]);
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

// ------------------------------------------------------------------ operand preparation

__device__ __forceinline__ void split16(float v, uint16_t& hi, uint16_t& lo) {
  const __half h = __float2half_rn(v);
  const __half l = __float2half_rn(v - __half2float(h));
  hi = __half_as_ushort(h);
  lo = __half_as_ushort(l);
}

// One warp per row: n = ||x|| (the norm the other dense-path kernels compute,
// in the same order), then [hi | lo] of 2^8 x / n.
template <typename T>
__global__ void __launch_bounds__(128) prep_rows_kernel(const T* __restrict__ x, int64_t ld, int d, int64_t seg_len,
                                                        int64_t seg_cap, int64_t row0, int64_t nrows,
                                                        uint16_t* __restrict__ a2, float* __restrict__ norms) {
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
  uint16_t* dst = a2 + w * (int64_t)(2 * d);
  for (int j = lane; j < d; j += 32) {
    uint16_t hi, lo;
    split16(to_f32(xr[j]) * inv * kSplitScale, hi, lo);
    dst[j] = hi;
    dst[d + j] = lo;
  }
  if (lane == 0) norms[(row / seg_len) * seg_cap + row % seg_len] = n;
}

// [hi | lo] of 2^8 r, two values per thread
__global__ void __launch_bounds__(256) split_rows_kernel(const float* __restrict__ r, int d, int64_t nrows,
                                                         uint16_t* __restrict__ a2) {
  const int64_t total = nrows * (int64_t)(d / 2);
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / (d / 2);
    const int j = 2 * (int)(e - row * (d / 2));
    const float2 v = *reinterpret_cast<const float2*>(r + row * d + j);
    uint16_t h0, l0, h1, l1;
    split16(v.x * kSplitScale, h0, l0);
    split16(v.y * kSplitScale, h1, l1);
    uint16_t* dst = a2 + row * (int64_t)(2 * d);
    *reinterpret_cast<uint32_t*>(dst + j) = (uint32_t)h0 | ((uint32_t)h1 << 16);
    *reinterpret_cast<uint32_t*>(dst + d + j) = (uint32_t)l0 | ((uint32_t)l1 << 16);
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled encode_tiled_fn() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
  });
  return fn;
}

// fp16 rows [rows][cols] (row stride ld elements), boxes of 64 columns x
// box_rows rows with the 128-byte swizzle; rows past `rows` read as zero
bool make_map(CUtensorMap* map, const uint16_t* base, int64_t cols, int64_t rows, int64_t ld, int box_rows) {
  PFN_cuTensorMapEncodeTiled enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool covers(int N, int K) { return N > 0 && K > 0 && N % kBN == 0 && K % kKC == 0; }

cudaError_t run(const Problem& p, unsigned* err, int num_sms, cudaStream_t st) {
  if (!covers(p.N, p.K) || p.nterms < 1 || p.nterms > 3 || p.M < 0 || p.M > INT32_MAX - kBM || !err)
    return cudaErrorInvalidValue;
  if (!aligned16(p.A) || !aligned16(p.B) || !aligned16(p.C) || (p.lda * 2) % 16 != 0 || (p.ldb * 2) % 16 != 0 ||
      p.ldc % 4 != 0)
    return cudaErrorInvalidValue;
  for (int t = 0; t < p.nterms; ++t)
    if (p.a_off[t] < 0 || p.a_off[t] % 8 != 0 || p.a_off[t] + p.K > p.lda || p.b_off[t] < 0 || p.b_off[t] % 8 != 0 ||
        p.b_off[t] + p.K > p.ldb)
      return cudaErrorInvalidValue;
  if (p.M == 0) return cudaSuccess;
  CUtensorMap am, bm;
  if (!make_map(&am, p.A, p.lda, p.M, p.lda, kBM) || !make_map(&bm, p.B, p.ldb, p.N, p.ldb, kBN))
    return cudaErrorInvalidValue;
  Args a{};
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.nterms = p.nterms;
  // distinct column ranges of A and of B, and which box each term reads
  int abase[3], bbase[3], ia[3] = {0, 0, 0}, ib[3] = {0, 0, 0};
  int na = 0, nbx = 0;
  for (int t = 0; t < p.nterms; ++t) {
    int i = 0;
    while (i < na && abase[i] != p.a_off[t]) ++i;
    if (i == na) abase[na++] = p.a_off[t];
    ia[t] = i;
    int j = 0;
    while (j < nbx && bbase[j] != p.b_off[t]) ++j;
    if (j == nbx) bbase[nbx++] = p.b_off[t];
    ib[t] = j;
  }
  if (na + nbx > kMaxBoxes) return cudaErrorInvalidValue;
  a.stages = std::min<int>(kMaxStages, (int)(kRing / ((uint32_t)(na + nbx) * kBoxBytes)));
  a.na = na;
  a.nb = nbx;
  a.a_base0 = abase[0];
  a.a_base1 = na > 1 ? abase[1] : 0;
  a.a_base2 = na > 2 ? abase[2] : 0;
  a.b_base0 = bbase[0];
  a.b_base1 = nbx > 1 ? bbase[1] : 0;
  a.b_base2 = nbx > 2 ? bbase[2] : 0;
  a.ia0 = ia[0], a.ia1 = ia[1], a.ia2 = ia[2];
  a.ib0 = ib[0], a.ib1 = ib[1], a.ib2 = ib[2];
  a.scale = p.scale;
  a.C = p.C;
  a.ldc = p.ldc;
  a.tiles_n = p.N / kBN;
  a.n_tiles = (p.M + kBM - 1) / kBM * a.tiles_n;
  a.err = err;
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int64_t ctas = std::min<int64_t>(a.n_tiles, (int64_t)num_sms);
  gemm_kernel<<<(unsigned)ctas, kThreads, kSmem, st>>>(am, bm, a);
  return cudaGetLastError();
}

cudaError_t prep_rows(int dt, const void* x, int64_t ld, int d, int64_t seg_len, int64_t seg_cap, int64_t row0,
                      int64_t nrows, uint16_t* a2, float* norms, cudaStream_t st) {
  if (nrows <= 0) return cudaSuccess;
  const unsigned blocks = (unsigned)ceil_div(nrows, 4);
  switch (dt) {
    case TQ_F32:
      prep_rows_kernel<float><<<blocks, 128, 0, st>>>((const float*)x, ld, d, seg_len, seg_cap, row0, nrows, a2, norms);
      break;
    case TQ_F16:
      prep_rows_kernel<__half><<<blocks, 128, 0, st>>>((const __half*)x, ld, d, seg_len, seg_cap, row0, nrows, a2,
                                                       norms);
      break;
    default:
      prep_rows_kernel<__nv_bfloat16><<<blocks, 128, 0, st>>>((const __nv_bfloat16*)x, ld, d, seg_len, seg_cap, row0,
                                                              nrows, a2, norms);
      break;
  }
  return cudaGetLastError();
}

cudaError_t split_rows(const float* r, int d, int64_t nrows, uint16_t* a2, cudaStream_t st) {
  if (nrows <= 0) return cudaSuccess;
  if (d % 2 != 0) return cudaErrorInvalidValue;
  const int64_t total = nrows * (int64_t)(d / 2);
  const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(total, 256), 148 * 16);
  split_rows_kernel<<<blocks, 256, 0, st>>>(r, d, nrows, a2);
  return cudaGetLastError();
}

void split_host(const float* v, int rows, int cols, uint16_t* out) {
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < cols; ++j) {
      const float s = v[(size_t)i * cols + j] * kSplitScale;
      const __half h = __float2half_rn(s);
      const __half l = __float2half_rn(s - __half2float(h));
      out[(size_t)i * 2 * cols + j] = __half_as_ushort(h);
      out[(size_t)i * 2 * cols + cols + j] = __half_as_ushort(l);
    }
}

}  // namespace gemm_tc
}  // namespace tq
