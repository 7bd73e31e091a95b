// Epilogue building blocks shared by the tensor-core kernels: vectorised
// loads / stores of 32-column row chunks and the fused residual + RMSNorm
// epilogue (LLaTTE notes, huaxiaozhuan.com, appendix A.2 display: post-norm
// Z = RMSNorm(R + MLA(R)), X = RMSNorm(Z + FFN(Z)); the FFN-down variant
// scatters each output row into the next layer's history / query rows).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace llatte {
namespace tc {

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 w = __ldg(s + j);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 f = __bfloat1622float2(h[k]);
      v[8 * j + 2 * k] = f.x;
      v[8 * j + 2 * k + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void add_f32x32(const float* src, float (&v)[32]) {
  const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float4 w = __ldg(s + j);
    v[4 * j] += w.x; v[4 * j + 1] += w.y; v[4 * j + 2] += w.z; v[4 * j + 3] += w.w;
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    d[j] = make_uint4(pack_bf16(v[8 * j], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                      pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
}

__device__ __forceinline__ void store_f32x32(float* dst, const float (&v)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 8; ++j) d[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

__device__ __forceinline__ void load_f16x32(const __half* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 w = __ldg(s + j);
    const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 f = __half22float2(h[k]);
      v[8 * j + 2 * k] = f.x;
      v[8 * j + 2 * k + 1] = f.y;
    }
  }
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store_f16x32(__half* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    d[j] = make_uint4(pack_f16(v[8 * j], v[8 * j + 1]), pack_f16(v[8 * j + 2], v[8 * j + 3]),
                      pack_f16(v[8 * j + 4], v[8 * j + 5]), pack_f16(v[8 * j + 6], v[8 * j + 7]));
}

// Residual chunk for columns [c, c + 32) of `row`, added to v (bf16 or fp16).
__device__ __forceinline__ void add_resid(const NormArgs& a, int64_t row, int N, int c,
                                          float (&v)[32]) {
  if (!a.resid) return;
  float r[32];
  if (a.resid_kind == RES_F16) load_f16x32((const __half*)a.resid + row * N + c, r);
  else load_bf16x32((const __nv_bfloat16*)a.resid + row * N + c, r);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] += r[i];
}

// Residual + RMSNorm epilogue of one 128-row tile whose accumulator holds the
// full row (BN == N columns, starting at taddr).  Two warps share each TMEM
// lane quadrant and take half of the columns each; their partial sums of
// squares meet in `red` ([2][128] floats) behind the group barrier `xbar`
// (bounded wait; returns false if the CTA is aborting).  Pass 1 reads the
// accumulator, adds the residual (read once) and stages the sum back in TMEM;
// pass 2 normalises, applies the gain and stores.
template <int BN>
__device__ __forceinline__ bool norm_epilogue(const NormArgs& a, uint32_t taddr, int64_t row,
                                              bool valid, int half, float* red, int rrow,
                                              uint64_t* xbar, uint32_t& xphase,
                                              volatile int* abort_flag, int32_t* status) {
  constexpr int HB = BN / 2;
  const int c0 = half * HB;
  const int N = BN;
  // pass 1: v = acc + residual, partial sum of squares; v goes back to TMEM.
  // The residual chunk is loaded (raw) before the TMEM read so that the two
  // latencies overlap.
  float ss = 0.f;
#pragma unroll 1
  for (int c = c0; c < c0 + HB; c += 32) {
    uint4 rr[4];
    const bool have = valid && a.resid;
    if (have) {
      const uint4* rp = reinterpret_cast<const uint4*>(
          (a.resid_kind == RES_F16 ? (const void*)((const __half*)a.resid + row * N + c)
                                   : (const void*)((const __nv_bfloat16*)a.resid + row * N + c)));
#pragma unroll
      for (int j = 0; j < 4; ++j) rr[j] = __ldg(rp + j);
    }
    float v[32];
    tmem_ld32(taddr + c, v);
    if (have) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f[4];
        if (a.resid_kind == RES_F16) {
          const __half2* h2 = reinterpret_cast<const __half2*>(&rr[j]);
#pragma unroll
          for (int k = 0; k < 4; ++k) f[k] = __half22float2(h2[k]);
        } else {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&rr[j]);
#pragma unroll
          for (int k = 0; k < 4; ++k) f[k] = __bfloat1622float2(h2[k]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[8 * j + 2 * k] += f[k].x;
          v[8 * j + 2 * k + 1] += f[k].y;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
    if (a.resid) tmem_st32(taddr + c, v);
  }
  red[half * 128 + rrow] = ss;
  if (!group_sync(xbar, xphase, abort_flag, status)) return false;
  ss += red[(half ^ 1) * 128 + rrow];
  const float inv = rsqrtf(ss / (float)N + a.eps);
  // destinations of this row
  __nv_bfloat16* d1 = nullptr;
  __nv_bfloat16* d2 = nullptr;
  float* f1 = nullptr;
  __half* r1 = nullptr;
  if (valid) {
    if (a.mode == NORM_PLAIN) {
      d1 = (__nv_bfloat16*)a.dst + row * N;
      if (a.dst_res) r1 = (__half*)a.dst_res + row * N;
    } else {
      const int u = a.row_user[row];
      const int64_t j = row - a.qoff_l[u];
      const int32_t nl = a.n_l[u];
      if (a.last) {
        if (a.final_rows) f1 = a.final_rows + row * N;
        else if (j >= nl) f1 = a.out + ((int64_t)u * a.n_q + (j - nl)) * N;
      } else {
        const int32_t nn = a.n_n[u];
        int64_t q = -1;
        if (j < nl) {
          d1 = (__nv_bfloat16*)a.Xh_n + (a.hoff_n[u] + j) * N;
          if (j >= nl - nn) q = a.qoff_n[u] + j - (nl - nn);
        } else {
          q = a.qoff_n[u] + nn + (j - nl);
        }
        if (q >= 0) {
          d2 = (__nv_bfloat16*)a.Xq_n + q * N;
          if (a.Xq_res_n) r1 = (__half*)a.Xq_res_n + q * N;
        }
      }
    }
  }
  // pass 2: normalise, scale by the gain, store
#pragma unroll 1
  for (int c = c0; c < c0 + HB; c += 32) {
    float g[32];
    load_bf16x32((const __nv_bfloat16*)a.g + c, g);
    float v[32];
    tmem_ld32(taddr + c, v);
    if (valid) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = v[i] * inv * g[i];
      if (d1) store_bf16x32(d1 + c, v);
      if (d2) store_bf16x32(d2 + c, v);
      if (f1) store_f32x32(f1 + c, v);
      if (r1) store_f16x32(r1 + c, v);
    }
  }
  return true;
}

}  // namespace tc
}  // namespace llatte
