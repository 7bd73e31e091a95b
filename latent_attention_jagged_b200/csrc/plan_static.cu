// llatte_plan_static: the pyramid plan of one batch without any device
// allocation.
//
// Some callers cannot call cudaMalloc at the point where they need the plan:
// code running inside another framework's memory pool, an allocator hook, or
// a process whose device memory is fully reserved up front.  For them this
// entry point keeps its scratch (per-layer history lengths, kept counts,
// offsets and totals) in one file-scope device array of fixed size, so the
// only memory it touches besides that array is the caller's own input and
// output buffers.
//
// The array lives on every GPU that loads the library until the process
// exits.  Its address is looked up once per device (cudaGetSymbolAddress) on
// the first call made with that device current; make that first call before
// any stream capture.  The address stays cached for the life of the process,
// so the call must not be used across a device reset (cudaDeviceReset or a
// primary-context reset), after which the array lives at a new address.  All calls on a device share the array, so calls whose
// executions overlap on the GPU (different streams, no ordering) race; order
// them on one stream or synchronise between them.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr int kMaxBatch = LLATTE_PLAN_STATIC_MAX_BATCH;
constexpr int kLayers = LLATTE_MAX_LAYERS + 1;  // + the virtual final layer
constexpr size_t kOffBytes = sizeof(int64_t) * kLayers * (kMaxBatch + 1);
constexpr size_t kCountBytes = sizeof(int32_t) * kLayers * kMaxBatch;
constexpr size_t kTotalsBytes = sizeof(int64_t) * 2 * kLayers;
constexpr size_t kWorkCountBytes = sizeof(int32_t) * 2 * kLayers;
constexpr size_t kScratchBytes = 2 * kOffBytes + 2 * kCountBytes + kTotalsBytes + kWorkCountBytes;

// hist_off | query_off | T | n | totals | work counters (each 8-byte aligned)
static __device__ __align__(256) unsigned char g_plan_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[64] = {};

// Device address of g_plan_scratch on the current device (looked up once).
void* scratch_address(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 64) { *err = cudaErrorInvalidDevice; return nullptr; }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_plan_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

// plan_out[l][0][u] = hist_off_l[u], plan_out[l][1][u] = query_off_l[u].
__global__ void copy_plan_kernel(const int64_t* __restrict__ hist, const int64_t* __restrict__ query,
                                 int64_t stride, int L, int B, int64_t* __restrict__ out) {
  const int64_t n = (int64_t)L * (B + 1);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int l = (int)(i / (B + 1));
    const int u = (int)(i % (B + 1));
    out[(int64_t)(2 * l) * (B + 1) + u] = hist[l * stride + u];
    out[(int64_t)(2 * l + 1) * (B + 1) + u] = query[l * stride + u];
  }
}

}  // namespace

extern "C" int llatte_plan_static(const llatte_dims* dims, const int64_t* offsets, int32_t B,
                                  int64_t* plan_out, int32_t* status_out, void* stream) {
  if (!dims || !offsets || !plan_out || !status_out) return LLATTE_ERR_ARG;
  const llatte_dims& D = *dims;
  if (D.n_layers < 1 || D.n_layers > LLATTE_MAX_LAYERS || D.n_q < 0 || D.max_len < 0 ||
      D.max_total < 0 || D.max_batch <= 0)
    return LLATTE_ERR_ARG;
  for (int l = 0; l < D.n_layers; ++l)
    if (D.keep[l] < 0 || (l && D.keep[l] > D.keep[l - 1])) return LLATTE_ERR_ARG;
  if (B < 0 || B > D.max_batch) return LLATTE_ERR_ARG;
  if (B > kMaxBatch) return LLATTE_ERR_UNSUPPORTED;   // beyond the fixed scratch
  cudaError_t err;
  unsigned char* base = (unsigned char*)scratch_address(&err);
  if (!base) return LLATTE_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(status_out, 0, sizeof(int32_t), s) != cudaSuccess) return LLATTE_ERR_CUDA;
  // B = 0 runs too: the plan of an empty batch is all zeros, and plan_out
  // gets them like any other batch's plan

  llatte::PlanDev p = {};
  p.stride = kMaxBatch + 1;
  p.hist_off = (int64_t*)base;
  p.query_off = (int64_t*)(base + kOffBytes);
  p.T = (int32_t*)(base + 2 * kOffBytes);
  p.n = (int32_t*)(base + 2 * kOffBytes + kCountBytes);
  p.totals = (int64_t*)(base + 2 * kOffBytes + 2 * kCountBytes);
  // attention work lists are not built here (the kernel is told so); the work
  // counters still get a home because a rejected batch clears them
  p.work_count = (int32_t*)(base + 2 * kOffBytes + 2 * kCountBytes + kTotalsBytes);
  p.work_next = p.work_count + kLayers;
  p.status = status_out;
  const int64_t max_total = D.max_total ? D.max_total : (int64_t)D.max_batch * D.max_len;
  if (llatte::launch_plan_on(p, D, max_total, offsets, B, s) != cudaSuccess) return LLATTE_ERR_CUDA;
  copy_plan_kernel<<<64, 256, 0, s>>>(p.hist_off, p.query_off, p.stride, D.n_layers, B, plan_out);
  if (cudaGetLastError() != cudaSuccess) return LLATTE_ERR_CUDA;
  return LLATTE_OK;
}
