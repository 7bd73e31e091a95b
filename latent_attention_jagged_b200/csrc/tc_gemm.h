// Interface of the tensor-core (tcgen05) kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

namespace llatte {

enum { TC_STORE = 0, TC_USERBIAS = 1, TC_SILU = 2, TC_NORM = 3, TC_F32 = 4 };

struct TcGemmParams {
  int64_t M_host;               // rows, unless M_dev != NULL
  const int64_t* M_dev;
  int64_t M_cap;                // largest M (sizes the grid)
  int N, K;
  __nv_bfloat16* D; int64_t ldd;                      // STORE / USERBIAS / SILU
  const float* bias; const int64_t* seg_off; int B;   // USERBIAS: bias[user(row), n]
  const int32_t* row_user;                             // user of each row
  NormArgs norm;                                       // NORM (acc unused)
  // F32: fp32 store, optionally one k-slice of a split-K sum (k_split slices
  // of the k-blocks) and one member of a batch of `groups` products.  Tile
  // (group g, rows m, columns n, slice s) reads A rows g * a_group_rows + m
  // and W rows g * w_group_rows + n, and writes
  // Dp[s * slice_stride + g * d_group_off + m * ldp + n]  (M, N per group).
  float* Dp; int64_t slice_stride; int k_split;
  int groups; int64_t a_group_rows; int w_group_rows; int64_t d_group_off; int64_t ldp;
  int32_t* status;
  int ab_f16;                   // A and the weight in fp16 (both operands of every MMA), else bf16
  int d_tma;                    // (set by the launcher) output stored by TMA boxes
};

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
// The same for an fp16 tensor.
bool make_tmap_f16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows);
bool tc_gemm_supported(int BN, int epi, int N, int K);
// d: a store map of the output (make_tmap_store16), or NULL: STORE / USERBIAS /
// SILU and a NORM_PLAIN epilogue with one output then write their rows as TMA
// boxes of 32 x 32 (rows past M up to the map's row count may be written).
cudaError_t launch_tc_gemm(int BN, int epi, const CUtensorMap& a, const CUtensorMap& b,
                           const TcGemmParams& p, int num_sms, cudaStream_t s,
                           const CUtensorMap* d = nullptr);
// Store map of a 16-bit [rows, cols] tensor for the epilogues: boxes of 32 rows x
// 32 columns with the 64-byte swizzle (the staging layout).  fp16 when f16.
bool make_tmap_store16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, bool f16);
// Residual + RMSNorm GEMM with N = 512 on pairs of SMs (256-row tiles); b_half:
// the weight with 128-row boxes (each CTA loads half of a k-block).
bool tc_gemm_pair_supported(int epi, int N, int K);
cudaError_t launch_tc_gemm_pair(int epi, const CUtensorMap& a, const CUtensorMap& b_half,
                                const TcGemmParams& p, int num_sms, cudaStream_t s);

}  // namespace llatte
