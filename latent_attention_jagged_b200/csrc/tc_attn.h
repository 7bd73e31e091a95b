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
  __nv_bfloat16* Ot;          // [sum q * heads, r]; per-head form: [sum q, heads * 64]
  int32_t* status;
  int inject_timeout;         // per-head kernel: every CTA's MMA issuer waits once on a barrier
                              //   that nothing arrives on (failure-detection test)
};

int attn_tc_keys(int r);
bool attn_tc_supported(int r);
cudaError_t launch_attn_tc(int r, const CUtensorMap& q, const CUtensorMap& c,
                           const AttnTcParams& p, int num_sms, cudaStream_t s);
// Per-head form (d_h = 64): q over [sum q, heads * 64] (128-row boxes), kv over
// [sum T, 2 * heads * 64] (K then V, 128-row boxes); work items (user,
// 128-row block * heads + head); two CTAs per SM.
cudaError_t launch_attn_heads(const CUtensorMap& q, const CUtensorMap& kv, const AttnTcParams& p,
                              int num_sms, cudaStream_t s);

}  // namespace llatte
