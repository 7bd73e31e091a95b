// Device evaluation of the FMA-pipe exponential that the attention softmax
// uses for a share of its probabilities, so that its arithmetic can be checked
// against the special-function unit and against exact values.
#include <cuda_runtime.h>
#include <stdint.h>

#include "llatte.h"
#include "tc_common.cuh"

namespace llatte {
namespace {

__global__ void exp2_eval_kernel(const float* __restrict__ x, float* __restrict__ y,
                                 float* __restrict__ y_hw, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i];
  const float b = i + 1 < n ? x[i + 1] : 0.f;
  const float2 r = tc::exp2_fma2(make_float2(a, b));
  y[i] = r.x;
  if (y_hw) y_hw[i] = tc::ex2_approx(a);
  if (i + 1 < n) {
    y[i + 1] = r.y;
    if (y_hw) y_hw[i + 1] = tc::ex2_approx(b);
  }
}

}  // namespace
}  // namespace llatte

extern "C" int llatte_exp2_eval(const float* x, float* y, float* y_hw, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return LLATTE_ERR_ARG;
  if (n == 0) return LLATTE_OK;
  const int threads = 256;
  const int64_t blocks = ((n + 1) / 2 + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return LLATTE_ERR_ARG;
  llatte::exp2_eval_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(x, y, y_hw, n);
  return cudaGetLastError() == cudaSuccess ? LLATTE_OK : LLATTE_ERR_CUDA;
}
