// Inner-product scores and fused top-k of many queries against a
// Q_prod-compressed set on the tcgen05 tensor cores (tq_score_tc.cu):
// coverage, workspace and launcher.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "tq_internal.h"

namespace tq {
namespace score_tc {

// Shapes covered: key codes of 1..3 bits whose odd-subset feature words come
// in groups of four (2^(k-1) d_pad / 32 a multiple of 4), m a multiple of
// 128, top-k of at most 32.
bool covers(const QParams& kp, int topk);

// Workspace bytes after the q' / u buffers: the query operand images and the
// per-item top-k candidates.
size_t workspace_bytes(const QParams& kp, int64_t nq, int64_t n_vec, int topk);

// Scores (scores != null: [nq][n_vec]) and / or the top-k per query (topk >
// 0: top_s, top_i [nq][topk], by score descending then index ascending) from
// the prepared queries qrot [nq][d_pad] and u [nq][m].  ws: workspace_bytes.
cudaError_t launch(const QParams& kp, const float* qrot, const float* u, int64_t nq, const uint32_t* codes,
                   const uint32_t* signs, const float* norms, const float* rnorms, int64_t n_vec, float* scores,
                   int topk, float* top_s, int64_t* top_i, void* ws, unsigned* err, int num_sms, cudaStream_t st);

}  // namespace score_tc
}  // namespace tq
