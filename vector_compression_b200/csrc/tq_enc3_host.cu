// Request checks, TMA descriptor and launch of the tensor-core encoder.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "tq_enc3.h"

namespace tq {
namespace enc3 {

namespace {

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

}  // namespace

bool try_encode(const QParams& qp, bool prod, const void* x, int dt, int64_t n_vec, int64_t ld,
                int64_t seg_len, int64_t seg_cap, int layout, uint32_t* codes, uint32_t* signs,
                float* norms, float* rnorms, unsigned* err_word, int num_sms, cudaStream_t st,
                cudaError_t* err) {
  const bool dp256 = !prod && qp.d_pad == 2 * kDP;  // Q_MSE at d_pad 256 (tq_encode3_256.cuh)
  if (qp.rot != TQ_ROT_HADAMARD || (qp.d_pad != kDP && !dp256)) return false;
  if (dt != TQ_F16 && dt != TQ_BF16) return false;
  if ((qp.d * 2) % 16 != 0 || (ld * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(x) & 15u) != 0)
    return false;
  if (seg_len <= 0 || seg_len % 32 != 0 || n_vec % seg_len != 0) return false;
  if (n_vec > ((int64_t)1 << 31) - 2 * kRows) return false;  // rows (and tile rows) < 2^31
  if (qp.k < 1 || qp.k > (prod ? 3 : 4)) return false;
  if (prod && qp.m != 64 && qp.m != 128) return false;
  if (!err_word) return false;
  if (n_vec == 0) {
    *err = cudaSuccess;
    return true;
  }
  PFN_cuTensorMapEncodeTiled enc = encode_tiled_fn();
  if (!enc) return false;
  // rows of d 16-bit values, row stride ld; boxes of 64 columns x 128 rows with
  // the 128-byte swizzle; columns d .. d_pad - 1 and rows past n_vec read as zero
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)qp.d, (cuuint64_t)n_vec};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  const cuuint32_t box[2] = {64, (cuuint32_t)kRows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(&map, dt == TQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         2, const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  Args a;
  a.n_vec = n_vec;
  a.seg_len = seg_len;
  a.seg_cap = seg_cap;
  a.seg_div = make_fastdiv((uint32_t)seg_len);
  a.n_tiles = (n_vec + kRows - 1) / kRows;
  a.codes = codes;
  a.signs = signs;
  a.norms = norms;
  a.rnorms = rnorms;
  a.err = err_word;
  const bool blk = layout == TQ_LAYOUT_BLOCK32;
  const int mode = prod ? MODE_PROD
                        : qp.unbiased ? (blk ? MODE_MSE_BLOCK_U : MODE_MSE_ROW_U)
                                      : (blk ? MODE_MSE_BLOCK : MODE_MSE_ROW);
  const int ctas = (int)std::min<int64_t>(a.n_tiles, (int64_t)num_sms);
  if (dp256)
    *err = dt == TQ_F16 ? launch256_f16(mode, map, qp, a, ctas, st) : launch256_bf16(mode, map, qp, a, ctas, st);
  else
    *err = dt == TQ_F16 ? launch_f16(mode, map, qp, a, ctas, st) : launch_bf16(mode, map, qp, a, ctas, st);
  return true;
}

}  // namespace enc3
}  // namespace tq
