// dense.h -- full causal prefill attention (the dense baseline), k_dense.cu.
#pragma once

#include "internal.h"

namespace qsa {

// bf16, 8 q heads per kv head, d = 128: out[b][r][h] = causal softmax attention
// of query row r (position q0 + r) over cached positions 0 .. q0 + r.
// q, out [B][n_q][8 Hkv][128]; k, v [B][kv_stride][Hkv][128].
cudaError_t launch_dense_prefill(const void *q, const void *k, const void *v, int B, int64_t n_q, int64_t q0,
                                 int64_t kv_stride, int Hkv, float scale, void *out, float *lse, unsigned *status,
                                 cudaStream_t s);

}  // namespace qsa
