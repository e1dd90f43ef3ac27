// 8-bit integer tensor-core decode attention (tq_attn3.cu): launcher.  The
// parameters and the partial-output format are in tq_attn_params.h.
#pragma once

#include <cuda_runtime.h>

#include "tq_attn_params.h"

namespace tq {
namespace attn3 {

// d_pad = 128 with m = 64 or 128 QJL rows, or d_pad = 256 with m = 256;
// 1..8 query heads per KV head, key codes of 1..3 bits, value codes of 1..4
// bits; grid = (chunks, groups), chunks a multiple of 64 tokens long.
cudaError_t launch(const attn::Params& p, int kk, int kv, int m, int dp, dim3 grid, cudaStream_t st);

}  // namespace attn3
}  // namespace tq
