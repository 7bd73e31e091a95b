// Attention-probability statistics of the query tokens of one layer (LLaTTE
// notes, huaxiaozhuan.com, appendix A.4 "Attention Weight Distribution":
// the cumulative attention on the most recent k events, on the k events with
// the largest weights, and the attention by hours before the request).
//
// One warp per (user, query token, head) row, after the layer's attention:
//   s_t   = q~ . c_t over the layer's history keys t (fp32 from the stored
//           absorbed query and latent rows; log2 units on the tensor-core
//           path, where log2(e) is folded into the query projection); the
//           lanes split the rank, so every key row is one coalesced read)
//   p_t   = softmax over t
//   recent[i] = sum of p over the 2^i most recent keys
//   hours[b]  = sum of p over keys with floor(age) = b (last bin: older too)
//   topk[i]   = sum of the 2^i largest p (bitonic sort of the row in shared
//               memory, descending)
// Sums across lanes use fixed shuffle trees; the hour bins add through
// shared-memory atomics.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace llatte {

namespace {

constexpr int kWarps = 4;

template <typename E, int RV>
__global__ void __launch_bounds__(32 * kWarps, 4) attn_export_kernel(ExportArgs a) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n2 = a.n2, r = a.r;
  // per warp: scores / probabilities [n2], hour bins [n_hours]
  float* sp = smem + (size_t)warp * (n2 + a.n_hours);
  float* sh = sp + n2;
  const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
  if (row >= (int64_t)a.B * a.n_q * a.heads) return;
  const int head = (int)(row % a.heads);
  const int64_t ui = row / a.heads;
  const int i = (int)(ui % a.n_q);
  const int u = (int)(ui / a.n_q);
  const int T = min(a.T[u], n2);     // n2 >= max_len; a rejected batch only loses values
  const int64_t m = a.qoff[u] + a.n[u] + i;             // the query token's row in the layer
  // lane l holds query coordinates l, l + 32, ... (RV = ceil(r / 32)); a
  // warp takes 32 keys at a time: every lane forms its partial dot products
  // with all 32 (each key row one coalesced read), then a transposed
  // reduction (31 shuffles) leaves key t0 + l's score in lane l
  const E* q = (const E*)a.Qt + m * a.q_row + head * a.q_head;
  float qv[RV];
#pragma unroll
  for (int j = 0; j < RV; ++j) {
    const int c = lane + 32 * j;
    qv[j] = c < r ? to_f(q[c]) : 0.f;
  }
  for (int b = lane; b < a.n_hours; b += 32) sh[b] = 0.f;
  const E* C = (const E*)a.C + a.hoff[u] * a.c_row + head * a.c_head;
  float mx = -INFINITY;
  for (int t0 = 0; t0 < T; t0 += 32) {
    float v[32];
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
      v[kk] = 0.f;
      if (t0 + kk < T) {
        const E* c = C + (int64_t)(t0 + kk) * a.c_row;
#pragma unroll
        for (int j = 0; j < RV; ++j) {
          const int cc = lane + 32 * j;
          if (cc < r) v[kk] = fmaf(qv[j], to_f(c[cc]), v[kk]);
        }
      }
    }
    // round with offset o: lanes with (lane & o) keep the upper half of the
    // remaining keys, the others the lower half; the halves swap and add
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int kk = 0; kk < o; ++kk) {
        const float send = up ? v[kk] : v[kk + o];
        const float keep = up ? v[kk + o] : v[kk];
        v[kk] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    // lane l now holds key t0 + l
    const int t = t0 + lane;
    if (t < T) {
      sp[t] = v[0];
      mx = fmaxf(mx, v[0]);
    }
  }
  mx = warp_max(mx);
  __syncwarp();
  for (int t = T + lane; t < n2; t += 32) sp[t] = -INFINITY;
  __syncwarp();
  float sum = 0.f;
  for (int t = lane; t < T; t += 32) {
    const float e = a.log2_scores ? exp2f(sp[t] - mx) : expf(sp[t] - mx);
    sp[t] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  const float inv = T > 0 ? 1.f / sum : 0.f;
  // probabilities; padding (t >= T) is 0, below every probability
  float rec[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) rec[k] = 0.f;
  const float* age = a.event_age ? a.event_age + a.evoff[u] + (a.T0[u] - T) : nullptr;
  for (int t = lane; t < n2; t += 32) {
    const float p = t < T ? sp[t] * inv : 0.f;
    sp[t] = p;
    if (t < T) {
      const int rho = T - t;                               // recency rank, 1 = most recent
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (k < a.n_k && rho <= (1 << k)) rec[k] += p;
      if (age) {
        const float ag = age[t];
        int b = ag >= (float)(a.n_hours - 1) ? a.n_hours - 1 : (int)floorf(fmaxf(ag, 0.f));
        atomicAdd(&sh[b], p);
      }
    }
  }
  const int64_t o = row * a.n_k;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (k >= a.n_k) break;
    const float v = warp_sum(rec[k]);
    if (lane == 0) a.recent[o + k] = v;
  }
  __syncwarp();
  if (a.hours)
    for (int b = lane; b < a.n_hours; b += 32) a.hours[row * a.n_hours + b] = sh[b];
  // bitonic sort, descending
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncwarp();
      for (int x = lane; x < n2; x += 32) {
        const int y = x ^ stride;
        if (y > x) {
          const float vx = sp[x], vy = sp[y];
          const bool desc = (x & size) == 0;
          if (desc ? vx < vy : vx > vy) { sp[x] = vy; sp[y] = vx; }
        }
      }
    }
  }
  __syncwarp();
  for (int k = 0; k < a.n_k; ++k) {
    const int kk = min(1 << k, n2);
    float s = 0.f;
    for (int x = lane; x < kk; x += 32) s += sp[x];
    s = warp_sum(s);
    if (lane == 0) a.topk[o + k] = s;
  }
}

}  // namespace

size_t attn_export_smem(int n2, int r, int n_hours) {
  (void)r;
  return sizeof(float) * kWarps * ((size_t)n2 + n_hours);
}

template <typename E, int RV>
cudaError_t launch_rv(const ExportArgs& a, size_t smem, unsigned blocks, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_export_kernel<E, RV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_export_kernel<E, RV><<<blocks, 32 * kWarps, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename E>
cudaError_t launch_e(const ExportArgs& a, size_t smem, unsigned blocks, cudaStream_t s) {
  switch ((a.r + 31) / 32) {
    case 1: return launch_rv<E, 1>(a, smem, blocks, s);
    case 2: return launch_rv<E, 2>(a, smem, blocks, s);
    case 3: case 4: return launch_rv<E, 4>(a, smem, blocks, s);
    case 5: case 6: case 7: case 8: return launch_rv<E, 8>(a, smem, blocks, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_export(int elem, const ExportArgs& a, cudaStream_t s) {
  const int64_t rows = (int64_t)a.B * a.n_q * a.heads;
  if (rows == 0) return cudaSuccess;
  const size_t smem = attn_export_smem(a.n2, a.r, a.n_hours);
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  if (elem == 4) return launch_e<float>(a, smem, blocks, s);
  return launch_e<__nv_bfloat16>(a, smem, blocks, s);
}

}  // namespace llatte
