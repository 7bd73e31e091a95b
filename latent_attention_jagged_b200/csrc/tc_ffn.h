// Interface of the fused tensor-core FFN kernel (d = 256).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "internal.h"

namespace llatte {

struct FfnTcParams {
  const int64_t* M_dev;   // rows (device)
  int64_t M_cap;          // largest M (sizes the grid)
  int F;                  // hidden width (multiple of 128)
  NormArgs norm;          // residual + RMSNorm + scatter of the output rows
  int32_t* status;
};

bool ffn_tc_supported(int d, int f);
cudaError_t launch_ffn_tc(const CUtensorMap& z, const CUtensorMap& w1, const CUtensorMap& w2,
                          const FfnTcParams& p, int num_sms, cudaStream_t s);

}  // namespace llatte
