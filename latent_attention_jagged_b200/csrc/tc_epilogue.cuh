// Epilogue building blocks shared by the tensor-core kernels: row staging
// through shared memory for row-contiguous global accesses, and the fused residual + RMSNorm
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

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- row staging
// A TMEM load leaves one accumulator row in each lane, but global memory is
// fastest when one instruction covers whole 32-byte sectors of few rows.  So
// rows pass through a per-warp shared-memory buffer of 32 rows x 64 bytes
// (kStageBytes): the 16-byte chunk k of row r sits at chunk k ^ ((r >> 1) & 3),
// which keeps both directions free of bank conflicts, and every global access
// then moves 8 rows x 64 bytes.  All 32 lanes must take part; a lane whose
// row has no source / destination passes a null pointer.
constexpr uint32_t kStageBytes = 32 * 64;

__device__ __forceinline__ uint32_t stage_slot(uint32_t stg, int r, int k) {
  return stg + (uint32_t)r * 64u + ((uint32_t)(k ^ ((r >> 1) & 3)) << 4);
}

// Lane l holds the 64 bytes x of row l; the row goes to lane l's `dst`.
__device__ __forceinline__ void stage_store(uint32_t stg, const uint4 (&x)[4], void* dst) {
  const int lane = threadIdx.x & 31, k = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) st_shared_v4(stage_slot(stg, lane, j), x[j]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2);
    char* d = reinterpret_cast<char*>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), r));
    const uint4 v = ld_shared_v4(stage_slot(stg, r, k));
    if (d) *reinterpret_cast<uint4*>(d + 16 * k) = v;
  }
  __syncwarp();
}

// The same 32 x 64-byte staging, stored by one bulk tensor copy instead of
// per-lane global stores: the staging layout (16-byte chunk k of row r at
// chunk k ^ ((r >> 1) & 3), buffer 512-byte aligned) is the 64-byte swizzle
// of a TMA box of 32 rows x 32 16-bit columns, so lane l's row goes to row
// y + l, columns x .. x + 31 of the map's tensor (rows past the tensor's end
// are dropped by the copy).  `store` false stages nothing to global memory
// (a box that lies wholly past the rows in use).  The buffer is reused only
// after the previous copy out of it has read it; call stage_tma_drain once
// after the last box.
__device__ __forceinline__ void stage_store_tma(uint32_t stg, const uint4 (&x)[4],
                                                const CUtensorMap* map, int32_t cx, int32_t cy,
                                                bool store) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) tma_store_wait_read();
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) st_shared_v4(stage_slot(stg, lane, j), x[j]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && store) {
    tma_store_2d(map, stg, cx, cy);
    tma_store_commit();
  }
}
__device__ __forceinline__ void stage_tma_drain() {
  if ((threadIdx.x & 31) == 0) tma_store_wait_all();
  __syncwarp();
}

// Global loads of the 64 bytes at lane r's `src` (zeros for a null pointer),
// 8 rows per instruction; stage_deliver then hands each lane its own row.
__device__ __forceinline__ void stage_fetch(const void* src, uint4 (&t)[4]) {
  const int lane = threadIdx.x & 31, k = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + (lane >> 2);
    const char* s = reinterpret_cast<const char*>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), r));
    t[i] = s ? __ldg(reinterpret_cast<const uint4*>(s + 16 * k)) : make_uint4(0, 0, 0, 0);
  }
}
__device__ __forceinline__ void stage_deliver(uint32_t stg, const uint4 (&t)[4], uint4 (&x)[4]) {
  const int lane = threadIdx.x & 31, k = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) st_shared_v4(stage_slot(stg, i * 8 + (lane >> 2), k), t[i]);
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = ld_shared_v4(stage_slot(stg, lane, j));
  __syncwarp();
}

__device__ __forceinline__ void pack_bf16x32(const float* v, uint4 (&x)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    x[j] = make_uint4(pack_bf16(v[8 * j], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                      pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
}

// Residual chunks of this thread's part of the row held in registers (the
// row's BN columns are split into P parts, one per warp of the lane
// quadrant): the first PD 32-column chunks are fetched before the accumulator
// is ready (their latency overlaps the wait); pass 1 refills each slot PD
// chunks ahead.
template <int BN, int PDMAX = 4, int P = 2>
struct NormPre {
  static constexpr int CH = BN / (32 * P);      // 32-column chunks per part
  static constexpr int PD = CH < PDMAX ? CH : PDMAX;   // chunks in flight
  uint4 t[PD][4];
};

template <int BN, int PDMAX, int P>
__device__ __forceinline__ void norm_prefetch(const NormArgs& a, int64_t row, bool valid,
                                              int part, NormPre<BN, PDMAX, P>& pre) {
  if (!a.resid) return;
  // a per-user residual (context term of a low-rank query) is row user(row)
  const int64_t res_row = (valid && a.resid_user) ? (int64_t)a.resid_user[row] : row;
  const char* src = valid ? (const char*)a.resid + (res_row * BN + part * (BN / P)) * 2 : nullptr;
#pragma unroll
  for (int i = 0; i < NormPre<BN, PDMAX, P>::PD; ++i)
    stage_fetch(src ? src + 64 * i : nullptr, pre.t[i]);
}

// Copy the RMSNorm gain (N bf16) into shared memory; every thread of the CTA
// calls this before the CTA's first barrier.
__device__ __forceinline__ void load_gain(const NormArgs& a, int N, __nv_bfloat16* sg) {
  for (int i = threadIdx.x; i < N / 8; i += blockDim.x)
    reinterpret_cast<uint4*>(sg)[i] = __ldg(reinterpret_cast<const uint4*>(a.g) + i);
}

// Residual + RMSNorm epilogue of one 128-row tile whose accumulator holds the
// full row (BN == N columns, starting at taddr).  P warps share each TMEM
// lane quadrant and take BN / P of the columns each; their partial sums of
// squares meet in `red` ([P][128] floats, added in part order so that every
// part gets the same sum) behind the group barrier `xbar`
// (bounded wait; returns false if the CTA is aborting).  Pass 1 reads the
// accumulator, adds the residual (read once, from the chunks `pre` holds and
// refills) and stages the sum back in TMEM; pass 2
// normalises, applies the gain (`sg`, in shared memory) and stores.  Global
// reads and writes go through the warp's staging buffer `stg`.  With `tmap`
// (NORM_PLAIN with a single output, dst or dst_res, of the map's type) the
// rows leave as TMA boxes of 32 rows (from row0) x 32 columns.
template <int BN, int PDMAX, int P>
__device__ __forceinline__ bool norm_epilogue(const NormArgs& a, uint32_t taddr, int64_t row,
                                              bool valid, int part, float* red, int rrow,
                                              uint64_t* xbar, uint32_t& xphase,
                                              volatile int* abort_flag, int32_t* status,
                                              uint32_t stg, NormPre<BN, PDMAX, P>& pre,
                                              const __nv_bfloat16* sg,
                                              const CUtensorMap* tmap = nullptr,
                                              int64_t row0 = 0) {
  constexpr int HB = BN / P;
  const int c0 = part * HB;
  const int N = BN;
  const bool have = a.resid != nullptr;
  const int64_t res_row = (valid && have && a.resid_user) ? (int64_t)a.resid_user[row] : row;
  const char* rsrc = (valid && have) ? (const char*)a.resid + (res_row * N) * 2 : nullptr;
  // pass 1: v = acc + residual, partial sum of squares; v goes back to TMEM.
  float ss = 0.f;
  constexpr int PD = NormPre<BN, PDMAX, P>::PD;
  // with one chunk in flight the loop need not be unrolled (the slot index is
  // always 0), which keeps register pressure down at four parts per row
#pragma unroll (PD == 1 ? 1 : NormPre<BN, PDMAX, P>::CH)
  for (int ci = 0; ci < NormPre<BN, PDMAX, P>::CH; ++ci) {
    const int c = c0 + 32 * ci;
    float v[32];
    tmem_ld32(taddr + c, v);
    if (have) {
      uint4 rr[4];
      stage_deliver(stg, pre.t[ci % PD], rr);
      if (ci + PD < NormPre<BN, PDMAX, P>::CH)
        stage_fetch(rsrc ? rsrc + 2 * (c + 32 * PD) : nullptr, pre.t[ci % PD]);
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
    if (have) tmem_st32(taddr + c, v);
  }
  red[part * 128 + rrow] = ss;
  if (!group_sync(xbar, xphase, abort_flag, status)) return false;
  ss = 0.f;
#pragma unroll
  for (int q = 0; q < P; ++q) ss += red[q * 128 + rrow];
  const float inv = rsqrtf(ss / (float)N + a.eps);
  // destinations of this row (null: none)
  __nv_bfloat16* d1 = nullptr;
  __nv_bfloat16* d2 = nullptr;
  float* f1 = nullptr;
  __half* r1 = nullptr;
  if (valid) {
    if (a.mode == NORM_PLAIN) {
      if (a.dst) d1 = (__nv_bfloat16*)a.dst + row * N;
      if (a.dst_res) r1 = (__half*)a.dst_res + row * N;
    } else {
      const int u = a.row_user[row];
      const int64_t j = row - a.qoff_l[u];
      const int32_t nl = a.n_l[u];
      if (a.last) {
        if (a.zraw) {
          if (j >= nl) d1 = (__nv_bfloat16*)a.zraw + ((int64_t)u * a.n_q + (j - nl)) * N;
        } else if (a.final_rows) {
          f1 = a.final_rows + row * N;
        } else if (j >= nl) {
          f1 = a.out + ((int64_t)u * a.n_q + (j - nl)) * N;
        }
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
          if (a.Xq_n) d2 = (__nv_bfloat16*)a.Xq_n + q * N;
          if (a.Xq_res_n) r1 = (__half*)a.Xq_res_n + q * N;
        }
      }
    }
  }
  const unsigned full = 0xffffffffu;
  const bool any_d1 = __any_sync(full, d1 != nullptr), any_d2 = __any_sync(full, d2 != nullptr);
  const bool any_f1 = __any_sync(full, f1 != nullptr), any_r1 = __any_sync(full, r1 != nullptr);
  const bool box_live = __any_sync(full, valid);
  // pass 2: normalise, scale by the gain, store
#pragma unroll 1
  for (int c = c0; c < c0 + HB; c += 32) {
    float v[32];
    tmem_ld32(taddr + c, v);
    {
      // the gain, 8 columns (one 16-byte shared-memory load) at a time
      const uint32_t ga = smem_u32(sg + c);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w = ld_shared_v4(ga + 16 * j);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h2[k]);
          v[8 * j + 2 * k] *= inv * f.x;
          v[8 * j + 2 * k + 1] *= inv * f.y;
        }
      }
    }
    uint4 x[4];
    if (tmap) {
      // one plain output: bf16 dst or the fp16 residual copy, by TMA
      if (a.dst) {
        pack_bf16x32(v, x);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          x[j] = make_uint4(pack_f16(v[8 * j], v[8 * j + 1]), pack_f16(v[8 * j + 2], v[8 * j + 3]),
                            pack_f16(v[8 * j + 4], v[8 * j + 5]), pack_f16(v[8 * j + 6], v[8 * j + 7]));
      }
      stage_store_tma(stg, x, tmap, c, (int32_t)row0, box_live);
      continue;
    }
    if (any_d1 || any_d2) {
      pack_bf16x32(v, x);
      if (any_d1) stage_store(stg, x, d1 ? d1 + c : nullptr);
      if (any_d2) stage_store(stg, x, d2 ? d2 + c : nullptr);
    }
    if (any_r1) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        x[j] = make_uint4(pack_f16(v[8 * j], v[8 * j + 1]), pack_f16(v[8 * j + 2], v[8 * j + 3]),
                          pack_f16(v[8 * j + 4], v[8 * j + 5]), pack_f16(v[8 * j + 6], v[8 * j + 7]));
      stage_store(stg, x, r1 ? r1 + c : nullptr);
    }
    if (any_f1) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          x[j] = make_uint4(__float_as_uint(v[16 * h + 4 * j]), __float_as_uint(v[16 * h + 4 * j + 1]),
                            __float_as_uint(v[16 * h + 4 * j + 2]),
                            __float_as_uint(v[16 * h + 4 * j + 3]));
        stage_store(stg, x, f1 ? f1 + c + 16 * h : nullptr);
      }
    }
  }
  return true;
}

}  // namespace tc
}  // namespace llatte
