// Residual + RMSNorm GEMM with N = 512 on pairs of SMs (cta_group::2):
//   D = RMSNorm(R + A W^T) with W [512, K]: the output projection
//   Z = RMSNorm(R + o~ (W_o W_uv)^T) and the FFN down-projection
//   X = RMSNorm(Z + W2 SiLU(W1 Z)) at d = 512 (LLaTTE notes, huaxiaozhuan.com,
//   appendix A.2 display and A.3).
//
// A 128 x 512 tile on one SM re-reads the whole weight matrix from L2 for
// every 128 rows; here two CTAs (one per SM) take 256-row tiles, rank 0 issues
// every MMA with M = 256, and each CTA loads its own 128 rows of A and HALF of
// each weight k-block (for the two 256-column MMA halves s, rows
// [256 s + 128 r, +128) in CTA r), so every weight byte crosses L2 and shared
// memory once per 256 rows.  Each CTA's TMEM holds its 128 rows x 512 fp32
// columns; its 8 epilogue warps run the residual + RMSNorm epilogue (plain or
// pyramid scatter) on them.  Completion of the pair MMAs reaches both CTAs by
// multicast commit; rank 1's "accumulator free" is forwarded to rank 0 by one
// thread with one remote arrival per tile.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tc_drain.cuh"
#include "tc_epilogue.cuh"
#include "tc_gemm.h"

namespace llatte {

using namespace tc;

namespace {

constexpr int BM = 128, BK = 64, BN = 512, NI = 256;
constexpr int kEpiWarps = 8;                        // two per TMEM lane quadrant
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;           // 16 KB: this CTA's 128 rows
constexpr uint32_t B_SUB = 128 * BK * 2;            // 16 KB: 128 weight rows of one half
constexpr uint32_t B_BYTES = 2 * B_SUB;             // this CTA's half of a k-block
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + 2 * 2 * 128 * 4 +
                        kEpiWarps * kStageBytes + BN * 2;
static_assert(SMEM <= 232448, "shared memory budget");

__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_norm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const TcGemmParams p) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = (uint64_t*)(sB + STAGES * B_BYTES);  // [STAGES] rank 0: both CTAs' bytes
  uint64_t* empty = full + STAGES;                        // [STAGES] both
  uint64_t* tfull = empty + STAGES;                       // both
  uint64_t* tempty_local = tfull + 1;                     // this CTA's epilogue done
  uint64_t* tempty_peer = tempty_local + 1;               // rank 0: rank 1's epilogue done
  uint64_t* drain = tempty_peer + 1;
  uint64_t* xbar = drain + 1;                             // epilogue group barrier
  uint32_t* tmem_slot = (uint32_t*)(xbar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* red = (float*)(smem + STAGES * STAGE_BYTES + 256);   // [2 tiles][2 halves][128]
  uint8_t* sStage = (uint8_t*)(red + 2 * 2 * 128);             // [epilogue warp][kStageBytes]
  __nv_bfloat16* sG = (__nv_bfloat16*)(sStage + kEpiWarps * kStageBytes);   // gain [BN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int KB = p.K / BK;
  const int kb0 = pair % KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(tempty_local, kEpiWarps);
    mbar_init(tempty_peer, 1);
    mbar_init(drain, 1);
    mbar_init(xbar, kEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  load_gain(p.norm, BN, sG);
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier kernels wrote
  pdl_wait();
  const int64_t M = p.M_dev ? *p.M_dev : p.M_host;
  const int64_t num_tiles = (M + 2 * BM - 1) / (2 * BM);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0;
      bool ok = true;
      for (int64_t t = pair; t < num_tiles && ok; t += n_pairs) {
        const int32_t arow = (int32_t)(t * 2 * BM + BM * rank);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          const uint32_t full_c = cluster_addr(&full[stage], 0);
          // k-blocks in a per-pair rotated order: the SMs do not all read the
          // same weight lines from L2 at the same moment
          const int kx = ((kb + kb0) % KB) * BK;
          tma_load_2d_pair(&tmA, full_c, sA + stage * A_BYTES, kx, arow);
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2)
            tma_load_2d_pair(&tmB, full_c, sB + stage * B_BYTES + s2 * B_SUB, kx,
                             s2 * NI + 128 * (int)rank);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // after an abort: rank 0's full barriers count both CTAs' bytes, and
      // the cluster barrier at the end holds rank 1 until rank 0 is past here
      if (rank == 0 && *abort_flag) drain_ring(full, STAGES, issued, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t IDESC = idesc_bf16(2 * BM, NI, false, false);
      int stage = 0;
      uint32_t phase = 0, ti = 0;
      bool ok = true;
      for (int64_t t = pair; t < num_tiles && ok; t += n_pairs, ++ti) {
        // both CTAs' epilogues have read the previous tile's accumulator
        if (!mbar_wait(tempty_local, (ti & 1) ^ 1, abort_flag, p.status) ||
            !mbar_wait_cluster(tempty_peer, (ti & 1) ^ 1, abort_flag, p.status))
          break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(a_addr + k * 32, 16, 1024);
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
              const uint64_t bd = sdesc_sw128(b_addr + s2 * B_SUB + k * 32, 16, 1024);
              umma_bf16_pair(tmem + s2 * NI, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(tfull);
      }
      // every pair MMA must be complete before either CTA releases TMEM
      umma_commit_pair(drain);
      int dummy = 0;
      mbar_wait(drain, 0, &dummy, p.status);
    } else if (lane == 0) {
      // rank 1: forward this CTA's "accumulator free" to rank 0
      const uint32_t peer_c = cluster_addr(tempty_peer, 0);
      uint32_t ti = 0;
      for (int64_t t = pair; t < num_tiles; t += n_pairs, ++ti) {
        if (!mbar_wait(tempty_local, ti & 1, abort_flag, p.status)) break;
        mbar_arrive_cluster(peer_c);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;      // which half of the columns
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int rr = q * 32 + lane;
    uint32_t ti = 0, xphase = 0;
    for (int64_t t = pair; t < num_tiles; t += n_pairs, ++ti) {
      const int64_t row = t * 2 * BM + BM * rank + rr;
      NormPre<BN, 4> pre;
      norm_prefetch(p.norm, row, row < M, half, pre);
      const bool ok = mbar_wait(tfull, ti & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (!norm_epilogue(p.norm, lane_base, row, row < M, half, red + (ti & 1) * 256, rr, xbar,
                         xphase, abort_flag, p.status,
                         smem_u32(sStage + (warp - 2) * kStageBytes), pre, sG))
        break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_local);
    }
  }
  __syncthreads();
  cluster_sync();          // rank 0's MMAs into both TMEMs are complete
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Pairs that can be resident at once (clusters of two CTAs of this kernel).
int max_pairs(int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev]) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_norm_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  n = std::min(n, num_sms / 2);
  if (dev < 64) cached[dev] = n;
  return n;
}

}  // namespace

bool tc_gemm_pair_supported(int epi, int N, int K) {
  return epi == TC_NORM && N == BN && K % BK == 0 && K > 0;
}

cudaError_t launch_tc_gemm_pair(int epi, const CUtensorMap& a, const CUtensorMap& b_half,
                                const TcGemmParams& p, int num_sms, cudaStream_t s) {
  if (!tc_gemm_pair_supported(epi, p.N, p.K)) return cudaErrorInvalidValue;
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_norm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  const int64_t max_tiles = (p.M_cap + 2 * BM - 1) / (2 * BM);
  const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(max_pairs(num_sms), max_tiles));
  return launch_dependent(gemm_pair_norm_kernel, dim3(2 * pairs), dim3(kThreads), SMEM, s, 2, a,
                          b_half, p);
}

}  // namespace llatte
