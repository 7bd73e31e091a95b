// Interface of the fused tensor-core FFN kernel (d = 256, pairs of SMs).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "internal.h"

namespace llatte {

struct FfnTcParams {
  const int64_t* M_dev;   // rows (device)
  int64_t M_cap;          // largest M (sizes the grid)
  int F;                  // hidden width (multiple of 128)
  int z_f16;              // Z and W1 in fp16 (both operands of the first product), else bf16
  NormArgs norm;          // residual + RMSNorm + scatter of the output rows
  int32_t* status;
};

bool ffn_tc_supported(int d, int f);
// X = RMSNorm(Z + W2 SiLU(W1 Z)) on pairs of SMs (cta_group::2, 256-row
// tiles).  w1h: W1 with 64-row boxes; w2h: W2 with 128-row boxes (each CTA
// loads half a chunk).  norm.mode NORM_SCATTER (the layer's FFN), or
// NORM_NONE: X = W2 SiLU(W1 Z) stored as bf16 rows to norm.dst (16-byte
// aligned; the output passes through fp16, so |X| must stay below 65504).
cudaError_t launch_ffn_pair(const CUtensorMap& z, const CUtensorMap& w1h, const CUtensorMap& w2h,
                            const FfnTcParams& p, int num_sms, cudaStream_t s);

}  // namespace llatte
