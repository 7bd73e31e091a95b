// CUDA-core (fp32 FFMA) kernels: the whole layer for the fp32 storage type,
// and the small steps (context bias, weight absorption, readout) for both.
//
// Layer equations (LLaTTE notes, huaxiaozhuan.com, appendix A.2 display and
// A.3 absorbed MLA; target-aware query from the daiwk.github.io notes):
//   KV    c_kv = RMSNorm_{g_kv}(X W_dkv^T)
//   Q     q~   = X W_qk^T + (c W_qkc^T)                 (per-user context bias)
//   ATTN  o~   = softmax(q~ . c_kv) c_kv over the visible keys
//   O     Z    = RMSNorm_{g1}(R + o~ W_ov^T)
//   FFN   X'   = RMSNorm_{g2}(Z + W2 SiLU(W1 Z))
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace llatte {

// ---------------------------------------------------------------- GEMM
// D[m, n] = sum_k A[m, k] * W[n, k]   (A [M, K] row-major, W [N, K] row-major)
// 64x64 tile, k-step 16, 256 threads, 4x4 outputs per thread.
constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

template <typename TA, typename TW, typename TD>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[SG_BK][SG_BM + 4];
  __shared__ float Ws[SG_BK][SG_BN + 4];
  const int64_t M = g.M_dev ? *g.M_dev : g.M_host;
  const int64_t m0 = (int64_t)blockIdx.y * SG_BM;
  const int n0 = blockIdx.x * SG_BN;
  if (m0 >= M) return;
  const TA* A = (const TA*)g.A;
  const TW* W = (const TW*)g.W;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += SG_BK) {
    for (int i = tid; i < SG_BM * SG_BK; i += 256) {
      int r = i / SG_BK, c = i % SG_BK;
      int64_t m = m0 + r;
      int k = k0 + c;
      As[c][r] = (m < M && k < g.K) ? to_f(A[m * g.lda + k]) : 0.f;
      int n = n0 + r;
      Ws[c][r] = (n < g.N && k < g.K) ? to_f(W[(int64_t)n * g.K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
    int u = 0;
    if (g.epi == EPI_USERBIAS || g.epi == EPI_USERBIAS_F32) u = segment_of(g.seg_off, g.B, m);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float v = acc[i][j];
      if (g.epi == EPI_USERBIAS || g.epi == EPI_USERBIAS_F32) v += g.bias[(int64_t)u * g.N + n];
      if (g.epi == EPI_SILU) v = silu_f(v);
      if (g.epi == EPI_F32 || g.epi == EPI_USERBIAS_F32) ((float*)g.D)[m * g.ldd + n] = v;
      else ((TD*)g.D)[m * g.ldd + n] = from_f<TD>(v);
    }
  }
}

template <typename TA, typename TW, typename TD>
static cudaError_t gemm3(const GemmArgs& g, cudaStream_t s) {
  dim3 grid((g.N + SG_BN - 1) / SG_BN, (unsigned)((g.M_max + SG_BM - 1) / SG_BM));
  if (grid.y == 0) return cudaSuccess;
  gemm_simt_kernel<TA, TW, TD><<<grid, 256, 0, s>>>(g);
  return cudaGetLastError();
}

cudaError_t launch_gemm_simt(int ea, int ew, int ed, const GemmArgs& g, cudaStream_t s) {
  typedef __nv_bfloat16 bf;
  if (ea == 4 && ew == 4) return gemm3<float, float, float>(g, s);
  if (ea == 2 && ew == 2 && ed == 2) return gemm3<bf, bf, bf>(g, s);
  if (ea == 2 && ew == 2 && ed == 4) return gemm3<bf, bf, float>(g, s);
  if (ea == 2 && ew == 4) return gemm3<bf, float, float>(g, s);
  if (ea == 4 && ew == 2) return gemm3<float, bf, float>(g, s);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- row norm
// v = acc + resid;  y = v / sqrt(mean(v^2) + eps) * g; one warp per row.
template <typename T>
__global__ void __launch_bounds__(256)
rownorm_kernel(NormArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t M = *a.M_dev;
  const int64_t m = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (m >= M) return;
  const int N = a.N;
  const float* row = a.acc + m * N;
  const T* g = (const T*)a.g;
  auto val = [&](int c) {
    float v = row[c];
    if (a.resid) {
      const int64_t i = (a.resid_user ? (int64_t)a.resid_user[m] : m) * N + c;
      if (a.resid_kind == RES_F32) v += ((const float*)a.resid)[i];
      else if (a.resid_kind == RES_F16) v += __half2float(((const __half*)a.resid)[i]);
      else v += to_f(((const T*)a.resid)[i]);
    }
    return v;
  };
  float ss = 0.f;
  for (int c = lane; c < N; c += 32) {
    float v = val(c);
    ss += v * v;
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / N + a.eps);
  // destinations
  T* d1 = nullptr;
  T* d2 = nullptr;
  float* f1 = nullptr;     // fp32 output row (final layer)
  void* r1 = nullptr;      // residual copy of this row
  if (a.mode == NORM_PLAIN) {
    d1 = (T*)a.dst + m * N;
    if (a.dst_res) r1 = a.dst_res;
  } else {
    const int u = segment_of(a.qoff_l, a.B, m);
    const int64_t j = m - a.qoff_l[u];
    const int32_t nl = a.n_l[u];
    if (a.last) {
      if (a.zraw) {
        if (j >= nl) d1 = (T*)a.zraw + ((int64_t)u * a.n_q + (j - nl)) * N;
      } else if (a.final_rows) {
        f1 = a.final_rows + m * N;
      } else if (j >= nl) {
        f1 = a.out + ((int64_t)u * a.n_q + (j - nl)) * N;
      }
    } else {
      const int32_t nn = a.n_n[u];
      int64_t q = -1;
      if (j < nl) {
        d1 = (T*)a.Xh_n + (a.hoff_n[u] + j) * N;
        if (j >= nl - nn) q = a.qoff_n[u] + j - (nl - nn);
      } else {
        q = a.qoff_n[u] + nn + (j - nl);
      }
      if (q >= 0) {
        d2 = (T*)a.Xq_n + q * N;
        if (a.Xq_res_n) r1 = a.Xq_res_n;
      }
    }
  }
  int64_t rrow = m;
  if (a.mode != NORM_PLAIN && d2) rrow = (d2 - (T*)a.Xq_n) / N;
  for (int c = lane; c < N; c += 32) {
    float y = val(c) * inv * to_f(g[c]);
    if (d1) d1[c] = from_f<T>(y);
    if (d2) d2[c] = from_f<T>(y);
    if (f1) f1[c] = y;
    if (r1) {
      if (a.res_kind == RES_F16) ((__half*)r1)[rrow * N + c] = __float2half_rn(y);
      else ((float*)r1)[rrow * N + c] = y;
    }
  }
}

cudaError_t launch_rownorm(int elem, const NormArgs& a, cudaStream_t s) {
  unsigned blocks = (unsigned)((a.M_max + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  if (elem == 4) rownorm_kernel<float><<<blocks, 256, 0, s>>>(a);
  else rownorm_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- attention
// One warp per (query row, head).  Lane i holds latent coordinates
// i, i+32, ...; online softmax over the visible keys of the row's user.
template <typename T, int RV>
__global__ void __launch_bounds__(256)
attn_simt_kernel(AttnArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t Mq = *a.Mq_dev;
  if (w >= Mq * a.heads) return;
  const int64_t m = w / a.heads;
  const int j = (int)(w % a.heads);
  const int u = segment_of(a.qoff, a.B, m);
  const int64_t jl = m - a.qoff[u];
  const int32_t Tu = a.T[u], n = a.n[u];
  const int64_t vis = jl < n ? (Tu - n + jl + 1) : Tu;
  const int r = a.r;
  const T* q = (const T*)a.Qt + (m * a.heads + j) * r;
  const T* C = (const T*)a.C + a.hoff[u] * r;
  float qv[RV], o[RV];
#pragma unroll
  for (int i = 0; i < RV; ++i) {
    int c = lane + 32 * i;
    qv[i] = c < r ? to_f(q[c]) : 0.f;
    o[i] = 0.f;
  }
  float mx = -INFINITY, l = 0.f;
  for (int64_t t = 0; t < vis; ++t) {
    const T* kr = C + t * r;
    float kv[RV];
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < RV; ++i) {
      int c = lane + 32 * i;
      kv[i] = c < r ? to_f(kr[c]) : 0.f;
      part = fmaf(qv[i], kv[i], part);
    }
    const float s = warp_sum(part);
    const float mn = fmaxf(mx, s);
    const float corr = __expf(mx - mn);
    const float pr = __expf(s - mn);
    l = l * corr + pr;
#pragma unroll
    for (int i = 0; i < RV; ++i) o[i] = fmaf(pr, kv[i], o[i] * corr);
    mx = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  T* out = (T*)a.Ot + (m * a.heads + j) * r;
#pragma unroll
  for (int i = 0; i < RV; ++i) {
    int c = lane + 32 * i;
    if (c < r) out[c] = from_f<T>(o[i] * inv);
  }
}

template <typename T>
static cudaError_t attn_t(const AttnArgs& a, cudaStream_t s) {
  unsigned blocks = (unsigned)((a.Mq_max * a.heads + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  if (a.r <= 32) attn_simt_kernel<T, 1><<<blocks, 256, 0, s>>>(a);
  else if (a.r <= 64) attn_simt_kernel<T, 2><<<blocks, 256, 0, s>>>(a);
  else if (a.r <= 128) attn_simt_kernel<T, 4><<<blocks, 256, 0, s>>>(a);
  else if (a.r <= 256) attn_simt_kernel<T, 8><<<blocks, 256, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(int elem, const AttnArgs& a, cudaStream_t s) {
  return elem == 4 ? attn_t<float>(a, s) : attn_t<__nv_bfloat16>(a, s);
}

// ---------------------------------------------------------------- context term
// bias[l][u][n] = sum_k c_u[k] W_qkc,l[k][n] for every layer at once: the
// per-user part of the absorbed target-aware query W_qk [x ; c] (daiwk.github.io
// notes, "core formula").  Block = (128 output columns, one layer, CTX_USERS
// users): the context rows sit in shared memory, each thread owns one column
// n and reads the weight rows W_qkc[k][n] coalesced.
constexpr int CTX_USERS = 8;
constexpr int CTX_COLS = 128;

template <typename T>
__global__ void __launch_bounds__(CTX_COLS)
ctx_bias_kernel(const T* __restrict__ ctx, CtxWeights w, int B, int dc,
                float* __restrict__ out, __half* __restrict__ out16) {
  extern __shared__ float cs[];                       // [CTX_USERS][dc]
  const int l = blockIdx.y;
  const int u0 = blockIdx.z * CTX_USERS;
  const int nu = min(CTX_USERS, B - u0);
  for (int i = threadIdx.x; i < CTX_USERS * dc; i += blockDim.x) {
    const int uu = i / dc, k = i % dc;
    cs[i] = uu < nu ? to_f(ctx[(int64_t)(u0 + uu) * dc + k]) : 0.f;
  }
  __syncthreads();
  const int n = blockIdx.x * CTX_COLS + threadIdx.x;
  const int hr = w.N[l];
  if (n >= hr) return;
  const float* W = w.W[l] + n;
  float acc[CTX_USERS] = {};
#pragma unroll 4
  for (int k = 0; k < dc; ++k) {
    const float wk = __ldg(W + (int64_t)k * hr);
#pragma unroll
    for (int uu = 0; uu < CTX_USERS; ++uu) acc[uu] = fmaf(cs[uu * dc + k], wk, acc[uu]);
  }
  for (int uu = 0; uu < nu; ++uu) {
    const int64_t o = w.off[l] + (int64_t)(u0 + uu) * hr + n;
    if (out16) out16[o] = __float2half_rn(acc[uu]);
    else out[o] = acc[uu];
  }
}

cudaError_t launch_ctx_bias(int elem, const void* ctx, const CtxWeights& w, int L, int B, int hr,
                            int dc, float* out, __half* out16, cudaStream_t s) {
  // hr: the widest layer; each layer's block uses its own width w.N[l]
  if (B == 0 || dc == 0) return cudaSuccess;
  dim3 grid((hr + CTX_COLS - 1) / CTX_COLS, L, (B + CTX_USERS - 1) / CTX_USERS);
  const size_t sm = sizeof(float) * CTX_USERS * dc;
  if (elem == 4)
    ctx_bias_kernel<float><<<grid, CTX_COLS, sm, s>>>((const float*)ctx, w, B, dc, out, out16);
  else
    ctx_bias_kernel<__nv_bfloat16><<<grid, CTX_COLS, sm, s>>>((const __nv_bfloat16*)ctx, w, B, dc,
                                                             out, out16);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- readout mean
// mean[u] = (1 / rows_u) sum of the user's final rows (zero for no rows).
// mean[u, :] = mean of user u's rows.  A block takes 128 columns (32 float4)
// of one user; its eight warps take every eighth row, four rows' loads in
// flight per warp (the sums of many rows in flight at once instead of one
// long dependent chain per column), then the eight partial sums are added in
// warp order (deterministic).  With mean16 set the mean is also written in
// bf16: the A operand of the tensor-core readout projection.
constexpr int kMeanWarps = 8;

__global__ void __launch_bounds__(32 * kMeanWarps)
mean_rows_kernel(const float* __restrict__ rows, const int64_t* __restrict__ qoff, int d,
                 float* __restrict__ mean, __nv_bfloat16* __restrict__ mean16) {
  __shared__ float4 part[kMeanWarps][32];
  const int u = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c4 = blockIdx.y * 32 + lane;                 // float4 column of this lane
  const int d4 = d / 4;
  const int64_t a = qoff[u], b = qoff[u + 1];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (c4 < d4) {
    const float4* r4 = reinterpret_cast<const float4*>(rows);
#pragma unroll 4
    for (int64_t i = a + warp; i < b; i += kMeanWarps) {
      const float4 v = __ldg(r4 + i * d4 + c4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && c4 < d4) {
    float4 t = part[0][lane];
    for (int w = 1; w < kMeanWarps; ++w) {
      const float4 p = part[w][lane];
      t.x += p.x; t.y += p.y; t.z += p.z; t.w += p.w;
    }
    const float inv = b > a ? 1.f / (float)(b - a) : 0.f;
    const float4 m = make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
    reinterpret_cast<float4*>(mean)[(int64_t)u * d4 + c4] = m;
    if (mean16) {
      const uint2 w = make_uint2(tc::pack_bf16(m.x, m.y), tc::pack_bf16(m.z, m.w));
      reinterpret_cast<uint2*>(mean16)[(int64_t)u * d4 + c4] = w;
    }
  }
}

cudaError_t launch_mean_rows(const float* rows, const int64_t* qoff, int B, int d, float* mean,
                             void* mean16, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  if (d % 4 != 0) return cudaErrorInvalidValue;
  mean_rows_kernel<<<dim3(B, (d / 4 + 31) / 32), 32 * kMeanWarps, 0, s>>>(
      rows, qoff, d, mean, (__nv_bfloat16*)mean16);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- summaries
// Sequence summaries (LLaTTE notes, appendix A.2 item 4), the steps after the
// bottleneck GEMM, which has left S partial sums per (user, bottleneck unit).
//   reduce  H[b, j] = SiLU(sum of the S partials of (b, j)), summed in slice
//           order so that the result does not depend on timing; one thread
//           per (b, j), eight partial loads in flight.  Written in fp32
//           [B, N], or in bf16 as the A operand of the batched tensor-core
//           output projection: [k][b_pad][rank]
//   up      out[b, k, i] = sum_t W_up,k[i, t] H[b, k * R + t]; a block takes
//           SUM_UB users, one summary and 256 outputs, with H of its users in
//           shared memory and the output projection stored transposed
//           ([t][i]: a warp reads 64 consecutive outputs' weights of one t in
//           one line); the weights of the next eight t are loaded while the
//           current eight are used
constexpr int SUM_UB = 8;

__global__ void __launch_bounds__(256) summary_reduce_kernel(SummaryArgs a) {
  // launched as a dependent of the bottleneck GEMM: the next kernel may start
  // its set-up at once; the partials are read only after the GEMM is complete
  tc::pdl_trigger();
  tc::pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= (int64_t)a.B * a.N) return;
  const float* p = a.P + i;
  float v = 0.f;
  int s = 0;
  for (; s + 8 <= a.S; s += 8) {
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = __ldcg(p + (int64_t)(s + q) * a.slice_stride);
#pragma unroll
    for (int q = 0; q < 8; ++q) v += x[q];
  }
  for (; s < a.S; ++s) v += __ldcg(p + (int64_t)s * a.slice_stride);
  v = silu_f(v);
  if (a.H) {
    a.H[i] = v;
  } else {
    const int64_t b = i / a.N;
    const int j = (int)(i - b * a.N), k = j / a.rank, t = j - k * a.rank;
    a.H16[((int64_t)k * a.b_pad + b) * a.rank + t] = __float2bfloat16_rn(v);
  }
}

__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

template <typename T>
__global__ void __launch_bounds__(128) summary_up_kernel(SummaryArgs a) {
  extern __shared__ float4 sh4[];                  // [SUM_UB][r8] fp32, zero padded
  float* sh = reinterpret_cast<float*>(sh4);
  const int b0 = blockIdx.x * SUM_UB, k = blockIdx.y;
  const int r = a.rank, r8 = (r + 7) & ~7;
  for (int idx = threadIdx.x; idx < SUM_UB * r8; idx += blockDim.x) {
    const int u = idx / r8, t = idx - u * r8;
    const int b = b0 + u;
    sh[idx] = (b < a.B && t < r) ? a.H[(int64_t)b * a.N + (int64_t)k * r + t] : 0.f;
  }
  __syncthreads();
  const int pi = blockIdx.z * blockDim.x + threadIdx.x;      // output pair
  if (pi >= a.d_seq / 2) return;
  const T* w = (const T*)a.Wt + (int64_t)k * r * a.d_seq + 2 * pi;
  float acc[SUM_UB][2];
#pragma unroll
  for (int u = 0; u < SUM_UB; ++u) acc[u][0] = acc[u][1] = 0.f;
  // t in groups of eight; rows t >= r read as zero weights
  auto fetch = [&](int t0, float2 (&wf)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      wf[i] = t0 + i < r ? load2(w + (int64_t)(t0 + i) * a.d_seq) : make_float2(0.f, 0.f);
  };
  float2 cur[8], nxt[8];
  fetch(0, cur);
#pragma unroll 1
  for (int t = 0; t < r8; t += 8) {
    if (t + 8 < r8) fetch(t + 8, nxt);
#pragma unroll
    for (int u = 0; u < SUM_UB; ++u) {
      const float4 h0 = sh4[(u * r8 + t) >> 2];
      const float4 h1 = sh4[((u * r8 + t) >> 2) + 1];
      const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[u][0] = fmaf(cur[i].x, hv[i], acc[u][0]);
        acc[u][1] = fmaf(cur[i].y, hv[i], acc[u][1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
  }
#pragma unroll
  for (int u = 0; u < SUM_UB; ++u) {
    const int b = b0 + u;
    if (b < a.B)
      *reinterpret_cast<float2*>(a.out + ((int64_t)b * a.n_sum + k) * a.d_seq + 2 * pi) =
          make_float2(acc[u][0], acc[u][1]);
  }
}

cudaError_t launch_summary_reduce(const SummaryArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  if (a.rank <= 0 || a.n_sum <= 0 || a.N != a.n_sum * a.rank || a.S < 1 ||
      (!a.H && (!a.H16 || a.b_pad < a.B)))
    return cudaErrorInvalidValue;
  const int64_t vals = (int64_t)a.B * a.N;
  return tc::launch_dependent(summary_reduce_kernel, dim3((unsigned)((vals + 255) / 256)),
                              dim3(256), 0, s, 1, a);
}

cudaError_t launch_summary_up(int elem, const SummaryArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  if (a.d_seq <= 0 || (a.d_seq & 1) || a.rank <= 0 || a.rank > 1024 || a.n_sum <= 0 || !a.H)
    return cudaErrorInvalidValue;
  const dim3 grid((a.B + SUM_UB - 1) / SUM_UB, a.n_sum, (a.d_seq / 2 + 127) / 128);
  const size_t smem = sizeof(float) * SUM_UB * ((a.rank + 7) & ~7);
  if (elem == 4) summary_up_kernel<float><<<grid, 128, smem, s>>>(a);
  else summary_up_kernel<__nv_bfloat16><<<grid, 128, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
__global__ void transpose_kernel(const T* __restrict__ src, int64_t rows, int64_t cols,
                                 T* __restrict__ dst) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= rows * cols) return;
  const int64_t r = i / cols, c = i - r * cols;
  dst[c * rows + r] = src[i];
}

// dst[i] = fp16(src[i]) for n bf16 values (exact in fp16's normal range: a
// bf16 mantissa fits in fp16's).
__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                                   int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = __float2half_rn(__bfloat162float(src[i]));
}

cudaError_t launch_bf16_to_f16(const void* src, void* dst, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4096);
  bf16_to_f16_kernel<<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16*)src, (__half*)dst, n);
  return cudaGetLastError();
}

cudaError_t launch_transpose(int elem, const void* src, int64_t rows, int64_t cols, void* dst,
                             cudaStream_t s) {
  const int64_t n = rows * cols;
  if (n <= 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (elem == 4) transpose_kernel<float><<<blocks, 256, 0, s>>>((const float*)src, rows, cols, (float*)dst);
  else transpose_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)src, rows, cols,
                                                                (__nv_bfloat16*)dst);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- absorption
// W_qk[j*r + a, k] = (qscale/sqrt(d_h)) sum_e W_uk[j*d_h + e, a] W_q[j*d_h + e, k]
//   (qscale = log2(e) when the attention kernel takes scores in log2 units)
//   (k < d -> W_qk in the storage type, k >= d -> W_qkc in fp32, stored
//    transposed as [d_ctx][h*r] so that the context kernel reads it coalesced)
// W_ov[n, j*r + a] = sum_e W_o[n, j*d_h + e] W_uv[j*d_h + e, a]
template <typename T>
__global__ void absorb_q_kernel(const T* W_q, const T* W_uk, int d, int dc, int heads, int dh,
                                int r, float qscale, T* W_qk, float* W_qkc) {
  // d here is the width of the query input (d, or q_rank for a low-rank query)
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int K = d + dc;
  if (idx >= (int64_t)heads * r * K) return;
  const int k = (int)(idx % K);
  const int row = (int)(idx / K);
  const int j = row / r, a = row % r;
  float s = 0.f;
  for (int e = 0; e < dh; ++e)
    s = fmaf(to_f(W_uk[(int64_t)(j * dh + e) * r + a]), to_f(W_q[(int64_t)(j * dh + e) * K + k]), s);
  s *= rsqrtf((float)dh) * qscale;
  if (k < d) W_qk[(int64_t)row * d + k] = from_f<T>(s);
  else W_qkc[(int64_t)(k - d) * heads * r + row] = s;
}

template <typename T>
__global__ void absorb_o_kernel(const T* W_o, const T* W_uv, int d, int heads, int dh, int r,
                                T* W_ov) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int HR = heads * r;
  if (idx >= (int64_t)d * HR) return;
  const int col = (int)(idx % HR);
  const int nrow = (int)(idx / HR);
  const int j = col / r, a = col % r;
  float s = 0.f;
  for (int e = 0; e < dh; ++e)
    s = fmaf(to_f(W_o[(int64_t)nrow * heads * dh + j * dh + e]), to_f(W_uv[(int64_t)(j * dh + e) * r + a]), s);
  W_ov[idx] = from_f<T>(s);
}

cudaError_t launch_absorb(int elem, const void* W_q, const void* W_uk, const void* W_uv,
                          const void* W_o, int d, int dq, int dc, int heads, int dh, int r,
                          float qscale, void* W_qk, float* W_qkc, void* W_ov, cudaStream_t s) {
  const int64_t nq = (int64_t)heads * r * (dq + dc), no = (int64_t)d * heads * r;
  const unsigned bq = (unsigned)((nq + 255) / 256), bo = (unsigned)((no + 255) / 256);
  if (elem == 4) {
    absorb_q_kernel<float><<<bq, 256, 0, s>>>((const float*)W_q, (const float*)W_uk, dq, dc, heads,
                                              dh, r, qscale, (float*)W_qk, W_qkc);
    absorb_o_kernel<float><<<bo, 256, 0, s>>>((const float*)W_o, (const float*)W_uv, d, heads, dh,
                                              r, (float*)W_ov);
  } else {
    typedef __nv_bfloat16 bf;
    absorb_q_kernel<bf><<<bq, 256, 0, s>>>((const bf*)W_q, (const bf*)W_uk, dq, dc, heads, dh, r,
                                           qscale, (bf*)W_qk, W_qkc);
    absorb_o_kernel<bf><<<bo, 256, 0, s>>>((const bf*)W_o, (const bf*)W_uv, d, heads, dh, r,
                                           (bf*)W_ov);
  }
  return cudaGetLastError();
}

template <typename T>
__global__ void split_ctx_cols_kernel(const T* __restrict__ src, int rows, int d, int dc,
                                      T* __restrict__ dst_x, float* __restrict__ dst_c,
                                      float scale) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const int K = d + dc;
  if (i >= (int64_t)rows * K) return;
  const int row = (int)(i / K), col = (int)(i % K);
  const float v = to_f(src[i]) * scale;          // one rounding into the storage type
  if (col < d) dst_x[(int64_t)row * d + col] = from_f<T>(v);
  else dst_c[(int64_t)(col - d) * rows + row] = v;
}

cudaError_t launch_split_ctx_cols(int elem, const void* src, int rows, int d, int dc, void* dst_x,
                                  float* dst_c, float scale, cudaStream_t s) {
  const int64_t n = (int64_t)rows * (d + dc);
  if (n <= 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (elem == 4)
    split_ctx_cols_kernel<float><<<blocks, 256, 0, s>>>((const float*)src, rows, d, dc,
                                                         (float*)dst_x, dst_c, scale);
  else
    split_ctx_cols_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        (const __nv_bfloat16*)src, rows, d, dc, (__nv_bfloat16*)dst_x, dst_c, scale);
  return cudaGetLastError();
}

}  // namespace llatte
