// Interface of the tensor-core latent-attention kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace llatte {

struct AttnTcParams {
  const int32_t* work;        // [2 * items]: (user, block) pairs, longest first
  const int32_t* work_count;  // items of this layer (device)
  int max_items;              // upper bound (sizes the grid)
  const int32_t *T, *n;       // per user: history rows (keys) and kept rows
  const int64_t *hoff, *qoff; // per user: first key row, first query row
  int n_q, heads;
  __nv_bfloat16* Ot;          // [sum q * heads, r]
  int32_t* status;
};

int attn_tc_keys(int r);
bool attn_tc_supported(int r);
cudaError_t launch_attn_tc(int r, const CUtensorMap& q, const CUtensorMap& c,
                           const AttnTcParams& p, int num_sms, cudaStream_t s);

}  // namespace llatte
