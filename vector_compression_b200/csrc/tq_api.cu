// libtq C ABI: argument validation and kernel dispatch.  This is the single
// CUDA translation unit of the library (the kernels live in the included
// headers), so the device error word has one definition.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "tq_attention.cuh"
#include "tq_attn_params.h"
#include "tq_attn3.h"
#include "tq_device.cuh"
#include "tq_encode.cuh"
#include "tq_encode2.cuh"
#include "tq_enc2_launch.h"
#include "tq_enc3.h"
#include "tq_gemm.cuh"
#include "tq_gemm_tc.h"
#include "tq_internal.h"
#include "tq_score_tc.h"
#include "tq_scores.cuh"
#include "tq_wait.cuh"

namespace tq {

// Error word set by kernels whose bounded waits expire; read and cleared by
// tq_sync_check.  Kernels in other translation units get its address.
__device__ unsigned int g_device_error = 0;

namespace {

// Address of the error word in the current context, looked up on every call
// (a cached address would go stale after cudaDeviceReset or a context switch).
unsigned* device_error_ptr() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess ? (unsigned*)p : nullptr;
}

// One CTA waits, with the kernels' bounded-wait helper in both of its forms
// (polling test_wait, suspending try_wait), on mbarriers that nothing
// arrives at; each expiry is recorded in the error word.
__global__ void wait_expiry_kernel(long long budget, unsigned* err) {
  __shared__ __align__(8) uint64_t bar[2];
  const uint32_t b0 = (uint32_t)__cvta_generic_to_shared(&bar[0]);
  const uint32_t b1 = (uint32_t)__cvta_generic_to_shared(&bar[1]);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b0));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b1));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // phase 0 of each needs one arrival, which never comes
  if (threadIdx.x == 0) bounded_wait<false>(b0, 0u, err, budget);
  if (threadIdx.x == 1) bounded_wait<true>(b1, 0u, err, budget);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline size_t dtype_size(int dt) { return dt == TQ_F32 ? 4 : 2; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// SM count of the current device, cached per device ordinal (a device's SM
// count does not change; the cache entries are written once, atomically).
int num_sms() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDev) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < kMaxDev) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <typename T, bool PROD>
cudaError_t encode_hadamard_dispatch(const QParams& qp, const T* x, int64_t ld, int64_t seg_len,
                                     int64_t seg_cap, int64_t n_seg, int layout, uint32_t* codes,
                                     uint32_t* signs, float* norms, float* rnorms,
                                     cudaStream_t st) {
  const int64_t bps = ceil_div(seg_len, 32);
  const int64_t tasks = n_seg * bps;
  if (tasks == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>(ceil_div(tasks, 4), (int64_t)num_sms() * 16);
  const int A = qp.d_pad / 32;
#define TQ_ENC(AA)                                                                          \
  case AA:                                                                                  \
    encode_hadamard_kernel<AA, T, PROD><<<(unsigned)blocks, 128, 0, st>>>(                  \
        qp, x, ld, seg_len, seg_cap, bps, tasks, layout, codes, signs, norms, rnorms);      \
    break;
  switch (A) {
    TQ_ENC(1)
    TQ_ENC(2)
    TQ_ENC(4)
    TQ_ENC(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef TQ_ENC
  return cudaGetLastError();
}

template <typename T>
cudaError_t encode_dense(const QParams& qp, bool prod, const T* x, int64_t ld, int64_t n_vec,
                         int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes,
                         uint32_t* signs, float* norms, float* rnorms, float* ws, int64_t chunk,
                         cudaStream_t st) {
  const int d = qp.d;
  float* xh = ws;                          // [chunk][d]
  float* y = ws + (size_t)chunk * d;       // [chunk][d]  (y, then r)
  float* z = y + (size_t)chunk * d;        // [chunk][m]
  int64_t row = 0;
  while (row < n_vec) {
    // a chunk never crosses a segment boundary and starts on a 32-block
    const int64_t s = row / seg_len, t = row % seg_len;
    const int64_t rows = std::min<int64_t>(chunk, seg_len - t);
    normalize_rows_kernel<T><<<(unsigned)ceil_div(rows, 4), 128, 0, st>>>(
        x, ld, d, seg_len, seg_cap, row, rows, xh, norms);
    cudaError_t e = gemm_abt_f32(xh, qp.Pi, y, (int)rows, d, d, st);
    if (e != cudaSuccess) return e;
    if (layout == TQ_LAYOUT_ROW)
      launch_quantize_rows_warp(qp, y, seg_len, seg_cap, row, rows, prod, codes, norms, rnorms, st);
    else
      quantize_rows_kernel<<<(unsigned)ceil_div(ceil_div(rows, 32), 4), 128, 0, st>>>(
          qp, y, seg_len, seg_cap, row, rows, layout, prod, codes, norms, rnorms);
    if (prod) {
      e = gemm_abt_f32(y, qp.S, z, (int)rows, qp.m, d, st);
      if (e != cudaSuccess) return e;
      pack_signs_kernel<<<(unsigned)ceil_div(rows, 4), 128, 0, st>>>(z, qp.m, seg_len, seg_cap,
                                                                     row, rows, signs);
    }
    (void)s;
    row += rows;
  }
  return cudaGetLastError();
}

constexpr int64_t kDenseChunk = 32768;

// The dense path on the tensor cores (split-precision products, see
// tq_gemm_tc.h): y = Pi x as three fp16 terms, z = S r as two; the other
// steps are the kernels above.  Covers d and m multiples of 128.
bool dense_tc_covers(const QParams& qp, bool prod) {
  return qp.rot == TQ_ROT_DENSE && qp.Pi2 && gemm_tc::covers(qp.d, qp.d) &&
         (!prod || (qp.S16 && gemm_tc::covers(qp.m, qp.d)));
}

cudaError_t encode_dense_tc(const QParams& qp, bool prod, const void* x, int dt, int64_t ld, int64_t n_vec,
                            int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                            float* norms, float* rnorms, float* ws, int64_t chunk, cudaStream_t st) {
  const int d = qp.d;
  uint16_t* a2 = reinterpret_cast<uint16_t*>(ws);  // [chunk][2 d] fp16: x, then r
  float* y = ws + (size_t)chunk * d;                // [chunk][d]  (y, then r)
  float* z = y + (size_t)chunk * d;                 // [chunk][m]
  unsigned* err = device_error_ptr();
  const int nsm = num_sms();
  int64_t row = 0;
  while (row < n_vec) {
    // a chunk never crosses a segment boundary and starts on a 32-block
    const int64_t t = row % seg_len;
    const int64_t rows = std::min<int64_t>(chunk, seg_len - t);
    cudaError_t e = gemm_tc::prep_rows(dt, x, ld, d, seg_len, seg_cap, row, rows, a2, norms, st);
    if (e != cudaSuccess) return e;
    gemm_tc::Problem g1{};
    g1.A = a2;
    g1.lda = 2 * d;
    g1.M = rows;
    g1.B = qp.Pi2;
    g1.ldb = 2 * d;
    g1.N = d;
    g1.K = d;
    g1.nterms = 3;  // hi.lo + lo.hi + hi.hi (the small terms first)
    g1.a_off[0] = 0, g1.b_off[0] = d;
    g1.a_off[1] = d, g1.b_off[1] = 0;
    g1.a_off[2] = 0, g1.b_off[2] = 0;
    g1.scale = 1.0f / (gemm_tc::kSplitScale * gemm_tc::kSplitScale);
    g1.C = y;
    g1.ldc = d;
    e = gemm_tc::run(g1, err, nsm, st);
    if (e != cudaSuccess) return e;
    // Q_prod: r goes straight into a2 as the split operand of z = S r (x's
    // split there has been consumed by the y product)
    if (layout == TQ_LAYOUT_ROW)
      launch_quantize_rows_warp(qp, y, seg_len, seg_cap, row, rows, prod, codes, norms, rnorms, st,
                                prod ? a2 : nullptr);
    else
      quantize_rows_kernel<<<(unsigned)ceil_div(ceil_div(rows, 32), 4), 128, 0, st>>>(
          qp, y, seg_len, seg_cap, row, rows, layout, prod, codes, norms, rnorms);
    if (prod) {
      if (layout != TQ_LAYOUT_ROW) {  // the task-per-32-rows quantizer wrote r over y
        e = gemm_tc::split_rows(y, d, rows, a2, st);
        if (e != cudaSuccess) return e;
      }
      gemm_tc::Problem g2{};
      g2.A = a2;
      g2.lda = 2 * d;
      g2.M = rows;
      g2.B = qp.S16;  // exact in fp16
      g2.ldb = d;
      g2.N = qp.m;
      g2.K = d;
      g2.nterms = 2;  // lo.S + hi.S (the small term first)
      g2.a_off[0] = d, g2.b_off[0] = 0;
      g2.a_off[1] = 0, g2.b_off[1] = 0;
      g2.scale = 1.0f / gemm_tc::kSplitScale;
      g2.C = z;
      g2.ldc = qp.m;
      e = gemm_tc::run(g2, err, nsm, st);
      if (e != cudaSuccess) return e;
      pack_signs_kernel<<<(unsigned)ceil_div(rows, 4), 128, 0, st>>>(z, qp.m, seg_len, seg_cap, row, rows, signs);
    }
    row += rows;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- thread-per-vector encode

// Returns true (and launches) when the thread-per-vector kernels cover the
// request: Hadamard rotation, d_pad 128 or 256, 16-byte input rows and, for
// Q_prod, m in {64, 128, 256}.
bool try_encode_v2(const QParams& qp, bool prod, const void* x, int dt, int64_t n_vec, int64_t ld,
                   int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                   float* norms, float* rnorms, cudaStream_t st, cudaError_t* err) {
  if (qp.rot != TQ_ROT_HADAMARD || (qp.d_pad != 128 && qp.d_pad != 256)) return false;
  const int esz = (int)dtype_size(dt);
  if ((qp.d * esz) % 16 != 0) return false;
  if (prod && qp.m != 64 && qp.m != 128 && qp.m != 256) return false;
  if (prod && qp.k > 3) return false;
  enc2::SignMasks sg;
  for (int j = 0; j < kMaxHadamard; ++j) sg.m[j] = 0;
  auto dbit = [&](int j) { return (qp.dmask[j / 32] >> (j % 32)) & 1u; };
  if (esz == 2) {
    for (int p = 0; p < qp.d_pad / 2; ++p) sg.m[p] = (dbit(2 * p) << 15) | (dbit(2 * p + 1) << 31);
  } else {
    for (int j = 0; j < qp.d_pad; ++j) sg.m[j] = dbit(j) << 31;
  }
  enc2::Args a;
  a.st.x = (const unsigned char*)x;
  a.st.ld_bytes = ld * esz;
  a.st.row_bytes = qp.d * esz;
  const int cpr = a.st.row_bytes / 16;
  a.st.pitch = (cpr + ((cpr % 2 == 0) ? 1 : 2)) * 16;
  a.seg_len = seg_len;
  a.seg_cap = seg_cap;
  a.bps = ceil_div(seg_len, 32);
  a.n_tasks = (n_vec / seg_len) * a.bps;
  a.codes = codes;
  a.signs = signs;
  a.norms = norms;
  a.rnorms = rnorms;
  const size_t s_bytes = prod ? (size_t)qp.m * qp.d_pad * 2 : 0;
  const size_t stage1 = (size_t)4 * 32 * a.st.pitch;
  a.nbuf = (s_bytes + 2 * stage1 <= 113 * 1024) ? 2 : 1;
  size_t smem = s_bytes + a.nbuf * stage1;
  if (smem > 220 * 1024) return false;
  int tmem_cols = 0;
  if (prod) {
    const int need = qp.d_pad + qp.m;
    tmem_cols = 32;
    while (tmem_cols < need) tmem_cols *= 2;
    // at most 512 / tmem_cols CTAs may share an SM; pad shared memory so no
    // more than that can be co-resident
    const int per_sm = 512 / tmem_cols;
    if (per_sm == 1 && smem < 120 * 1024) smem = 120 * 1024;
  }
  a.tmem_cols = tmem_cols;
  if (a.n_tasks == 0) {
    *err = cudaSuccess;
    return true;
  }
  const int64_t want = ceil_div(a.n_tasks, 4);
  const int resident = (smem <= 113 * 1024) ? 2 : 1;
  const int ctas = (int)std::min<int64_t>(want, (int64_t)num_sms() * resident);
  const bool blk = layout == TQ_LAYOUT_BLOCK32;
  const int mode = prod ? enc2::MODE_PROD
                        : qp.unbiased ? (blk ? enc2::MODE_MSE_BLOCK_U : enc2::MODE_MSE_ROW_U)
                                      : (blk ? enc2::MODE_MSE_BLOCK : enc2::MODE_MSE_ROW);
  a.err = device_error_ptr();
  if (!a.err) return false;
  cudaError_t e;
  switch (dt) {
    case TQ_F32: e = enc2::launch_f32(qp.d_pad, mode, qp, sg, a, smem, ctas, st); break;
    case TQ_F16: e = enc2::launch_f16(qp.d_pad, mode, qp, sg, a, smem, ctas, st); break;
    default: e = enc2::launch_bf16(qp.d_pad, mode, qp, sg, a, smem, ctas, st); break;
  }
  *err = e;
  return true;
}

size_t encode_workspace_bytes(const QParams& qp, bool prod, int64_t n_vec) {
  if (qp.rot != TQ_ROT_DENSE || n_vec == 0) return 0;
  const int64_t chunk = std::min<int64_t>(kDenseChunk, round_up(n_vec, 32));
  return round_up((size_t)chunk * (2 * qp.d + (prod ? qp.m : 0)) * sizeof(float), 256);
}

}  // namespace

// Encoder selection: the tensor-core encoder whenever it covers a request,
// else the thread-per-vector one (f32 rows, d_pad 256), else the
// warp-per-vector kernels (any other shape).
int launch_encode(const QParams& qp, bool prod, const void* x, int dt, int64_t n_vec, int64_t ld,
                  int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                  float* norms, float* rnorms, void* ws, void* stream) {
  const int64_t n_seg = n_vec / seg_len;
  cudaStream_t st = S(stream);
  {
    cudaError_t e2;
    if (enc3::try_encode(qp, prod, x, dt, n_vec, ld, seg_len, seg_cap, layout, codes,
                                        signs, norms, rnorms, device_error_ptr(), num_sms(), st, &e2))
      return e2;
    if (try_encode_v2(qp, prod, x, dt, n_vec, ld, seg_len, seg_cap, layout, codes,
                                     signs, norms, rnorms, st, &e2))
      return e2;
  }
  if (qp.rot == TQ_ROT_DENSE) {
    const int64_t chunk = std::min<int64_t>(kDenseChunk, round_up(n_vec, 32));
    float* w = (float*)ws;
    if (dense_tc_covers(qp, prod))
      return encode_dense_tc(qp, prod, x, dt, ld, n_vec, seg_len, seg_cap, layout, codes, signs, norms, rnorms, w,
                             chunk, st);
    switch (dt) {
      case TQ_F32: return encode_dense(qp, prod, (const float*)x, ld, n_vec, seg_len, seg_cap, layout, codes, signs, norms, rnorms, w, chunk, st);
      case TQ_F16: return encode_dense(qp, prod, (const __half*)x, ld, n_vec, seg_len, seg_cap, layout, codes, signs, norms, rnorms, w, chunk, st);
      default: return encode_dense(qp, prod, (const __nv_bfloat16*)x, ld, n_vec, seg_len, seg_cap, layout, codes, signs, norms, rnorms, w, chunk, st);
    }
  }
#define TQ_DT(T)                                                                                  \
  return prod ? encode_hadamard_dispatch<T, true>(qp, (const T*)x, ld, seg_len, seg_cap, n_seg,   \
                                                  layout, codes, signs, norms, rnorms, st)        \
              : encode_hadamard_dispatch<T, false>(qp, (const T*)x, ld, seg_len, seg_cap, n_seg,  \
                                                   layout, codes, signs, norms, rnorms, st);
  switch (dt) {
    case TQ_F32: TQ_DT(float)
    case TQ_F16: TQ_DT(__half)
    default: TQ_DT(__nv_bfloat16)
  }
#undef TQ_DT
}

int launch_decode(const QParams& qp, int layout, const uint32_t* codes, const uint32_t* signs,
                  const float* norms, const float* rnorms, int64_t n_vec, int64_t seg_len,
                  int64_t seg_cap, float* out, int64_t ldo, void* stream) {
  cudaStream_t st = S(stream);
  const unsigned blocks = (unsigned)ceil_div(n_vec, 4);
  if (qp.rot == TQ_ROT_DENSE) {
    decode_dense_kernel<<<blocks, 128, 4 * qp.d * sizeof(float), st>>>(
        qp, layout, codes, signs, norms, rnorms, n_vec, seg_len, seg_cap, out, ldo);
    return cudaGetLastError();
  }
  switch (qp.d_pad / 32) {
#define TQ_DEC(AA)                                                                             \
  case AA:                                                                                     \
    decode_hadamard_kernel<AA><<<blocks, 128, 0, st>>>(qp, layout, codes, signs, norms, rnorms, \
                                                       n_vec, seg_len, seg_cap, out, ldo);     \
    break;
    TQ_DEC(1)
    TQ_DEC(2)
    TQ_DEC(4)
    TQ_DEC(8)
#undef TQ_DEC
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int launch_query_prep(const QParams& qp, const float* q, int64_t nq, int64_t ldq, float* qrot,
                      float* u, void* stream) {
  cudaStream_t st = S(stream);
  if (nq == 0) return cudaSuccess;
  if (qp.rot == TQ_ROT_DENSE) {
    // q' = Pi q and u = S q' as tiled GEMMs over all queries (rows of up to
    // 2^20 queries per launch keep the grid inside its limits)
    if (ldq > INT32_MAX) return cudaErrorInvalidValue;
    for (int64_t r0 = 0; r0 < nq; r0 += (int64_t)1 << 20) {
      const int rows = (int)std::min<int64_t>(nq - r0, (int64_t)1 << 20);
      float* qr = qrot + r0 * qp.d;
      cudaError_t e = gemm_abt_f32(q + r0 * ldq, qp.Pi, qr, rows, qp.d, qp.d, st, (int)ldq);
      if (e == cudaSuccess && u) e = gemm_abt_f32(qr, qp.S, u + r0 * qp.m, rows, qp.m, qp.d, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  // one query per block while that leaves SMs idle, four (sharing the S^T
  // loads) once there are many
  const bool four = nq >= (int64_t)num_sms() * 4;
  const unsigned qblocks = (unsigned)ceil_div(nq, four ? 4 : 1);
  const unsigned qthreads = qp.m >= 256 ? 256 : 128;  // threads over the m outputs of u
  switch (qp.d_pad / 32) {
#define TQ_QP(AA)                                                                                \
  case AA:                                                                                       \
    if (four)                                                                                    \
      query_prep_hadamard_kernel<AA, 4><<<qblocks, qthreads, 0, st>>>(qp, q, nq, ldq, qrot, u);  \
    else                                                                                         \
      query_prep_hadamard_kernel<AA, 1><<<qblocks, qthreads, 0, st>>>(qp, q, nq, ldq, qrot, u);  \
    break;
    TQ_QP(1)
    TQ_QP(2)
    TQ_QP(4)
    TQ_QP(8)
#undef TQ_QP
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

namespace {
int score_query_tile(const QParams& qp) {
  const size_t per_q = (size_t)(qp.d_pad + qp.m) * sizeof(float);
  int qt = (int)std::min<size_t>(32, (96 * 1024) / per_q);
  return std::max(qt, 1);
}
}  // namespace

int launch_scores(const QParams& qp, const float* qrot, const float* u, int64_t nq,
                  const uint32_t* codes, const uint32_t* signs, const float* norms,
                  const float* rnorms, int64_t n_vec, float* scores, void* stream) {
  if (nq == 0 || n_vec == 0) return cudaSuccess;
  const int qt = score_query_tile(qp);
  const size_t smem = (size_t)qt * (qp.d_pad + qp.m) * sizeof(float);
  // function attributes are per device: set on every call (a cheap host call)
  cudaError_t ae = cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 100 * 1024);
  if (ae != cudaSuccess) return ae;
  dim3 grid((unsigned)ceil_div(n_vec, kScoreThreads), (unsigned)ceil_div(nq, qt));
  scores_kernel<<<grid, kScoreThreads, smem, S(stream)>>>(qp, qrot, u, nq, qt, codes, signs, norms,
                                                          rnorms, n_vec, scores);
  return cudaGetLastError();
}

int launch_topk(const float* scores, int64_t nq, int64_t n_vec, int topk, float* top_s,
                int64_t* top_i, void* stream) {
  if (nq == 0) return cudaSuccess;
  topk_kernel<<<(unsigned)nq, kTopkThreads, 0, S(stream)>>>(scores, n_vec, topk, top_s, top_i);
  return cudaGetLastError();
}

size_t attention_workspace(const QParams& kp, const QParams& vp, int L, int B, int Hq, int Hkv,
                           int64_t seq, int* chunk_out, int* n_chunks_out) {
  const int64_t groups = (int64_t)L * B * Hkv;
  const int G = Hq / Hkv;
  // about 28 CTAs per SM in all (seven waves of the int8 kernel's four CTAs
  // per SM), rounding the chunk count down so the last wave stays full
  const int64_t target = (int64_t)num_sms() * 28;
  int64_t n_chunks = std::max<int64_t>(1, target / std::max<int64_t>(groups, 1));
  int64_t chunk = round_up(ceil_div(seq, n_chunks), 64);
  if (chunk < 1024) {
    // short chunks would spend most of a CTA on its per-query setup: aim at
    // one wave of CTAs instead (four per SM at d_pad 128; at d_pad 256, whose
    // CTAs run one per SM, two, measured 8% faster than four on a 128K-token
    // cache of 8 groups)
    const int64_t per_sm = kp.d_pad > 128 ? 2 : 4;
    n_chunks = std::max<int64_t>(1, (int64_t)num_sms() * per_sm / std::max<int64_t>(groups, 1));
    chunk = round_up(ceil_div(seq, n_chunks), 64);
  }
  chunk = std::max<int64_t>(chunk, 256);
  n_chunks = ceil_div(seq, chunk);
  if (chunk_out) *chunk_out = (int)chunk;
  if (n_chunks_out) *n_chunks_out = (int)n_chunks;
  const int64_t nq = (int64_t)L * B * Hq;
  size_t bytes = round_up((size_t)nq * kp.d_pad * 4, 256) + round_up((size_t)nq * kp.m * 4, 256) +
                 round_up((size_t)groups * n_chunks * G * (vp.d_pad + 2) * 4, 256);
  return bytes;
}

// The int8 tensor-core kernel (tq_attn3.cu) covers at most 8 query heads per
// KV head, key codes of 1..3 bits and value codes of 1..4 bits at d_pad = 128
// with m = 64 or 128 and at d_pad = 256 with m = 256, with the norm and sign
// arrays 16-byte aligned (it stages them with bulk copies); the SIMT kernel
// (tq_attention.cuh) covers every other shape.
static bool attn3_covers(const QParams& kp, const QParams& vp, int G, const void* ksigns,
                         const void* knorms, const void* krnorms, const void* vnorms) {
  const bool shape = (kp.d_pad == 128 && vp.d_pad == 128 && (kp.m == 128 || kp.m == 64)) ||
                     (kp.d_pad == 256 && vp.d_pad == 256 && kp.m == 256);
  return kp.rot == TQ_ROT_HADAMARD && shape && G >= 1 && G <= 8 && kp.k >= 1 && kp.k <= 3 &&
         vp.k >= 1 && vp.k <= 4 && aligned16(ksigns) && aligned16(knorms) && aligned16(krnorms) &&
         aligned16(vnorms);
}

int launch_decode_attention(const QParams& kp, const QParams& vp, const float* q, int L, int B,
                            int Hq, int Hkv, int64_t seq, int64_t cap, float scale,
                            const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                            const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                            float* out, void* ws, void* stream) {
  cudaStream_t st = S(stream);
  int chunk = 0, n_chunks = 0;
  attention_workspace(kp, vp, L, B, Hq, Hkv, seq, &chunk, &n_chunks);
  const int64_t nq = (int64_t)L * B * Hq;
  char* w = (char*)ws;
  float* qrot = (float*)w;
  w += round_up((size_t)nq * kp.d_pad * 4, 256);
  float* u = (float*)w;
  w += round_up((size_t)nq * kp.m * 4, 256);
  float* part = (float*)w;
  int e = launch_query_prep(kp, q, nq, kp.d, qrot, u, stream);
  if (e != cudaSuccess) return e;
  AttnShape sh;
  sh.G = Hq / Hkv;
  sh.groups = L * B * Hkv;
  sh.n_chunks = n_chunks;
  sh.chunk = chunk;
  sh.seq = seq;
  sh.cap = cap;
  sh.scale = scale;
  if (attn3_covers(kp, vp, sh.G, ksigns, knorms, krnorms, vnorms)) {
    attn::Params p2;
    p2.G = sh.G;
    p2.chunk = chunk;
    p2.n_chunks = n_chunks;
    p2.seq = seq;
    p2.cap = cap;
    p2.scale = scale;
    p2.kappa = kp.kappa;
    p2.qrot = qrot;
    p2.u = u;
    p2.kcodes = kcodes;
    p2.ksigns = ksigns;
    p2.knorms = knorms;
    p2.krnorms = krnorms;
    p2.kr16 = kp.rnorm_f16;
    p2.vcodes = vcodes;
    p2.vnorms = vnorms;
    p2.part = part;
    p2.err = device_error_ptr();
    attn::odd_feature_coefs(kp.centroids, kp.k, p2.kalpha, &p2.kalpha_sum);
    attn::odd_feature_coefs(vp.centroids, vp.k, p2.valpha, &p2.valpha_sum);
    const dim3 grid((unsigned)n_chunks, (unsigned)sh.groups);
    const cudaError_t ce = attn3::launch(p2, kp.k, vp.k, kp.m, kp.d_pad, grid, st);
    if (ce != cudaSuccess) return ce;
  } else {
  const size_t smem = (size_t)sh.G * (kp.d_pad + kp.m) * sizeof(float);
  // function attributes are per device: set on every call (a cheap host call)
  cudaError_t ae = cudaFuncSetAttribute(kp.d_pad <= 128 ? attention_chunk_kernel<1> : attention_chunk_kernel<2>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
  if (ae != cudaSuccess) return ae;
  dim3 grid((unsigned)n_chunks, (unsigned)sh.groups);
  if (kp.d_pad <= 128)
    attention_chunk_kernel<1><<<grid, kAttnThreads, smem, st>>>(kp, vp, sh, qrot, u, kcodes, ksigns, knorms, krnorms, vcodes, vnorms, part);
  else
    attention_chunk_kernel<2><<<grid, kAttnThreads, smem, st>>>(kp, vp, sh, qrot, u, kcodes, ksigns, knorms, krnorms, vcodes, vnorms, part);
  cudaError_t ce = cudaGetLastError();
  if (ce != cudaSuccess) return ce;
  }
  const unsigned cblocks = (unsigned)((int64_t)sh.groups * sh.G);  // one per (group, head)
  switch (vp.d_pad / 32) {
#define TQ_CMB(AA)                                                                                 \
  case AA:                                                                                         \
    attention_combine_hadamard_kernel<AA><<<cblocks, 256, 0, st>>>(vp, sh, part, out, Hq, Hkv);    \
    break;
    TQ_CMB(1)
    TQ_CMB(2)
    TQ_CMB(4)
    TQ_CMB(8)
#undef TQ_CMB
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int read_and_clear_device_error(void* stream, unsigned* err) {
  cudaError_t e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return e;
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  *err = v;
  return e;
}

}  // namespace tq

// ====================================================================== C ABI

namespace {

tq_status cuda_status(int e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

tq_status check_segments(int64_t n_vec, int64_t* seg_len, int64_t* seg_cap, bool block) {
  if (n_vec < 0) return TQ_ERR_INVALID_ARG;
  if (*seg_len == 0) *seg_len = n_vec;
  if (*seg_len < 0) return TQ_ERR_INVALID_ARG;
  if (n_vec == 0) return TQ_OK;
  if (n_vec % *seg_len != 0) return TQ_ERR_INVALID_ARG;
  if (*seg_cap == 0) *seg_cap = block ? (*seg_len + 31) / 32 * 32 : *seg_len;
  if (*seg_cap < *seg_len) return TQ_ERR_INVALID_ARG;
  if (block && *seg_cap % 32 != 0) return TQ_ERR_INVALID_ARG;
  return TQ_OK;
}

tq_status check_encode_common(const tq_params* p, const void* x, tq_dtype dt, int64_t n_vec,
                              int64_t ld, int64_t* seg_len, int64_t* seg_cap, int layout) {
  if (!p) return TQ_ERR_INVALID_ARG;
  if (dt != TQ_F32 && dt != TQ_F16 && dt != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (layout != TQ_LAYOUT_ROW && layout != TQ_LAYOUT_BLOCK32) return TQ_ERR_INVALID_ARG;
  tq_status s = check_segments(n_vec, seg_len, seg_cap, layout == TQ_LAYOUT_BLOCK32);
  if (s != TQ_OK) return s;
  if (n_vec == 0) return TQ_OK;
  if (!x || ld < p->q.d) return TQ_ERR_INVALID_ARG;
  if (!tq::aligned16(x) || (ld * (int64_t)tq::dtype_size(dt)) % 16 != 0) return TQ_ERR_INVALID_ARG;
  if (p->q.rot == TQ_ROT_DENSE && layout == TQ_LAYOUT_BLOCK32 && *seg_len % 32 != 0)
    return TQ_ERR_UNSUPPORTED;
  return TQ_OK;
}

}  // namespace

extern "C" {

tq_status tq_encode_workspace_size(const tq_params* p, int64_t n_vec, size_t* bytes) {
  if (!p || !bytes || n_vec < 0) return TQ_ERR_INVALID_ARG;
  *bytes = tq::encode_workspace_bytes(p->q, p->mode == TQ_MODE_PROD, n_vec);
  return TQ_OK;
}

tq_status tq_encode_mse(const tq_params* p, const void* x, tq_dtype dt, int64_t n_vec, int64_t ld,
                        int64_t seg_len, int64_t seg_cap, tq_layout layout, uint32_t* codes,
                        float* norms, void* ws, size_t ws_bytes, void* stream) {
  tq_status s = check_encode_common(p, x, dt, n_vec, ld, &seg_len, &seg_cap, layout);
  if (s != TQ_OK) return s;
  if (p->mode != TQ_MODE_MSE && p->mode != TQ_MODE_MSE_UNBIASED) return TQ_ERR_INVALID_ARG;
  if (n_vec == 0) return TQ_OK;
  if (!codes || !norms || !tq::aligned16(codes) || !tq::aligned16(norms)) return TQ_ERR_INVALID_ARG;
  const size_t need = tq::encode_workspace_bytes(p->q, false, n_vec);
  if (need > 0 && (!ws || ws_bytes < need || !tq::aligned256(ws))) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_encode(p->q, false, x, dt, n_vec, ld, seg_len, seg_cap, layout,
                                       codes, nullptr, norms, nullptr, ws, stream));
}

tq_status tq_encode_prod(const tq_params* p, const void* x, tq_dtype dt, int64_t n_vec, int64_t ld,
                         int64_t seg_len, int64_t seg_cap, uint32_t* codes, uint32_t* signs,
                         float* norms, float* rnorms, void* ws, size_t ws_bytes, void* stream) {
  tq_status s = check_encode_common(p, x, dt, n_vec, ld, &seg_len, &seg_cap, TQ_LAYOUT_ROW);
  if (s != TQ_OK) return s;
  if (p->mode != TQ_MODE_PROD) return TQ_ERR_INVALID_ARG;
  if (n_vec == 0) return TQ_OK;
  if (!codes || !signs || !norms || !rnorms) return TQ_ERR_INVALID_ARG;
  if (!tq::aligned16(codes) || !tq::aligned16(signs) || !tq::aligned16(norms) || !tq::aligned16(rnorms))
    return TQ_ERR_INVALID_ARG;
  const size_t need = tq::encode_workspace_bytes(p->q, true, n_vec);
  if (need > 0 && (!ws || ws_bytes < need || !tq::aligned256(ws))) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_encode(p->q, true, x, dt, n_vec, ld, seg_len, seg_cap,
                                       TQ_LAYOUT_ROW, codes, signs, norms, rnorms, ws, stream));
}

tq_status tq_decode(const tq_params* p, tq_layout layout, const uint32_t* codes,
                    const uint32_t* signs, const float* norms, const float* rnorms, int64_t n_vec,
                    int64_t seg_len, int64_t seg_cap, float* out, int64_t ldo, void* stream) {
  if (!p) return TQ_ERR_INVALID_ARG;
  if (layout != TQ_LAYOUT_ROW && layout != TQ_LAYOUT_BLOCK32) return TQ_ERR_INVALID_ARG;
  tq_status s = check_segments(n_vec, &seg_len, &seg_cap, layout == TQ_LAYOUT_BLOCK32);
  if (s != TQ_OK) return s;
  if (n_vec == 0) return TQ_OK;
  if (!codes || !norms || !out || ldo < p->q.d) return TQ_ERR_INVALID_ARG;
  if (signs && (p->mode != TQ_MODE_PROD || !rnorms)) return TQ_ERR_INVALID_ARG;
  if (!tq::aligned16(codes) || !tq::aligned16(norms) || !tq::aligned16(out)) return TQ_ERR_INVALID_ARG;
  return cuda_status(tq::launch_decode(p->q, layout, codes, signs, norms, rnorms, n_vec, seg_len,
                                       seg_cap, out, ldo, stream));
}

tq_status tq_scores_workspace_size(const tq_params* kp, int64_t nq, int64_t n_vec, int topk,
                                   size_t* bytes) {
  if (!kp || !bytes || nq < 0 || n_vec < 0 || topk < 0) return TQ_ERR_INVALID_ARG;
  size_t b = tq::round_up((size_t)nq * kp->q.d_pad * 4, 256) + tq::round_up((size_t)nq * kp->q.m * 4, 256);
  if (tq::score_tc::covers(kp->q, topk))
    b += tq::score_tc::workspace_bytes(kp->q, nq, n_vec, topk);  // no score matrix: the top-k is fused
  else if (topk > 0)
    b += tq::round_up((size_t)nq * n_vec * 4, 256);
  *bytes = b;
  return TQ_OK;
}

tq_status tq_scores(const tq_params* kp, const float* q, int64_t nq, int64_t ldq,
                    const uint32_t* codes, const uint32_t* signs, const float* norms,
                    const float* rnorms, int64_t n_vec, float* scores, int topk, float* top_s,
                    int64_t* top_i, void* ws, size_t ws_bytes, void* stream) {
  if (!kp || kp->mode != TQ_MODE_PROD) return TQ_ERR_INVALID_ARG;
  if (nq < 0 || n_vec < 0 || topk < 0 || topk > tq::kTopkMax) return TQ_ERR_INVALID_ARG;
  if (!scores && topk == 0) return TQ_ERR_INVALID_ARG;
  if (topk > 0 && (!top_s || !top_i || topk > n_vec)) return TQ_ERR_INVALID_ARG;
  if (nq == 0 || n_vec == 0) return TQ_OK;
  if (!q || ldq < kp->q.d || !codes || !signs || !norms || !rnorms) return TQ_ERR_INVALID_ARG;
  size_t need = 0;
  tq_scores_workspace_size(kp, nq, n_vec, topk, &need);
  if (!ws || ws_bytes < need || !tq::aligned256(ws)) return TQ_ERR_WORKSPACE;
  char* w = (char*)ws;
  float* qrot = (float*)w;
  w += tq::round_up((size_t)nq * kp->q.d_pad * 4, 256);
  float* u = (float*)w;
  w += tq::round_up((size_t)nq * kp->q.m * 4, 256);
  int e = tq::launch_query_prep(kp->q, q, nq, ldq, qrot, u, stream);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  // the tensor-core scorer (fused top-k) whenever it covers the shape
  if (tq::score_tc::covers(kp->q, topk)) {
    if (!tq::aligned16(signs) || !tq::aligned16(codes)) return TQ_ERR_INVALID_ARG;
    e = tq::score_tc::launch(kp->q, qrot, u, nq, codes, signs, norms, rnorms, n_vec, scores, topk, top_s, top_i, w,
                             tq::device_error_ptr(), tq::num_sms(), tq::S(stream));
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
  }
  float* full = topk > 0 ? (float*)w : scores;
  e = tq::launch_scores(kp->q, qrot, u, nq, codes, signs, norms, rnorms, n_vec, full, stream);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  if (topk > 0) {
    if (scores && scores != full) {
      e = cudaMemcpyAsync(scores, full, (size_t)nq * n_vec * 4, cudaMemcpyDeviceToDevice,
                          tq::S(stream));
      if (e != cudaSuccess) return TQ_ERR_CUDA;
    }
    e = tq::launch_topk(full, nq, n_vec, topk, top_s, top_i, stream);
    if (e != cudaSuccess) return TQ_ERR_CUDA;
  }
  return TQ_OK;
}

tq_status tq_decode_attention_workspace_size(const tq_params* kp, const tq_params* vp, int L,
                                             int B, int Hq, int Hkv, int64_t seq,
                                             size_t* bytes) {
  if (!kp || !vp || !bytes || L < 1 || B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || seq < 1)
    return TQ_ERR_INVALID_ARG;
  *bytes = tq::attention_workspace(kp->q, vp->q, L, B, Hq, Hkv, seq, nullptr, nullptr);
  return TQ_OK;
}

tq_status tq_decode_attention(const tq_params* kp, const tq_params* vp, const float* q, int L,
                              int B, int Hq, int Hkv, int64_t seq, int64_t cap, float scale,
                              const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                              const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                              float* out, void* ws, size_t ws_bytes, void* stream) {
  if (!kp || !vp || kp->mode != TQ_MODE_PROD || (vp->mode != TQ_MODE_MSE && vp->mode != TQ_MODE_MSE_UNBIASED))
    return TQ_ERR_INVALID_ARG;
  if (kp->q.d != vp->q.d || kp->q.rot != vp->q.rot) return TQ_ERR_INVALID_ARG;
  if (kp->q.rot != TQ_ROT_HADAMARD) return TQ_ERR_UNSUPPORTED;
  if (L < 1 || B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0) return TQ_ERR_INVALID_ARG;
  if (Hq / Hkv > tq::kAttnMaxG) return TQ_ERR_UNSUPPORTED;
  if (seq < 1 || cap < seq || cap % 32 != 0) return TQ_ERR_INVALID_ARG;
  if (!q || !kcodes || !ksigns || !knorms || !krnorms || !vcodes || !vnorms || !out)
    return TQ_ERR_INVALID_ARG;
  if (!tq::aligned16(q) || !tq::aligned16(kcodes) || !tq::aligned16(vcodes) || !tq::aligned16(out))
    return TQ_ERR_INVALID_ARG;
  size_t need = tq::attention_workspace(kp->q, vp->q, L, B, Hq, Hkv, seq, nullptr, nullptr);
  if (!ws || ws_bytes < need || !tq::aligned256(ws)) return TQ_ERR_WORKSPACE;
  return cuda_status(tq::launch_decode_attention(kp->q, vp->q, q, L, B, Hq, Hkv, seq, cap, scale,
                                                 kcodes, ksigns, knorms, krnorms, vcodes, vnorms,
                                                 out, ws, stream));
}

tq_status tq_check_wait_expiry(int64_t budget_cycles, void* stream) {
  if (budget_cycles < 1 || budget_cycles > (int64_t(1) << 31)) return TQ_ERR_INVALID_ARG;
  unsigned* err = tq::device_error_ptr();
  if (!err) return TQ_ERR_CUDA;
  tq::wait_expiry_kernel<<<1, 32, 0, tq::S(stream)>>>((long long)budget_cycles, err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_sync_check(void* stream) {
  unsigned err = 0;
  if (tq::read_and_clear_device_error(stream, &err) != cudaSuccess) return TQ_ERR_CUDA;
  if (err == 0) return TQ_OK;
  return err == TQ_ERR_TIMEOUT ? TQ_ERR_TIMEOUT : TQ_ERR_INTERNAL;
}

}  // extern "C"
