// Tensor-core GEMM for sm_100a: D[m, n] = sum_k A[m, k] W[n, k] (bf16 in,
// fp32 accumulation in TMEM) with the layer's epilogues fused.
//
// Roles (576 threads, one CTA per SM, persistent over 128 x BN tiles):
//   warp 0      TMA producer: A (128 x 64) and W (BN x 64) k-blocks into a
//               STAGES-deep ring of 128-byte-swizzled shared-memory tiles
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (128 x NI x 16) and
//               commits stage releases / accumulator-ready events
//   warps 2..17 epilogue, four warps per TMEM lane quadrant, each taking a
//               quarter of the tile's columns (a half for BN = 64; then two of
//               the four idle): TMEM -> registers (tcgen05.ld), then one of
//               STORE     bf16 store
//               USERBIAS  + per-user context term (absorbed query projection)
//               SILU      SiLU (FFN up-projection)
//               F32       fp32 store (a split-K slice's partial sums, or one
//                         member of a batch of products)
//               NORM      + residual (read once: the sum is staged back in
//                         TMEM), RMSNorm over the full row (BN == N; the
//                         parts' sums of squares meet in shared memory),
//                         store bf16 (+ fp16 residual copy) or scatter into the
//                         next layer's history / query rows (pyramid trimming)
// The accumulator is double-buffered in TMEM when 2 * BN <= 512 columns, so
// the epilogue of tile i overlaps the MMAs of tile i + 1.  With F32 a tile is
// (group, row block, column block, k-slice); the slices of one output tile
// are consecutive tile indices.
//
// Equations (LLaTTE notes, huaxiaozhuan.com, appendix A.2 display and A.3):
// KV latent RMSNorm(X W_down^KV); absorbed query X (W_uk^T W_q)^T + context
// term; Z = RMSNorm(R + o~ (W_o W_uv)^T); FFN W2 SiLU(W1 Z) + Z, RMSNorm.
// F32: the sequence summaries (appendix A.2 item 4): the bottleneck
// projection, whose K = n_q * d is long and whose output is small (split-K),
// and the per-summary output projections (a batch of products).
#include <cuda.h>
#include <cuda_fp16.h>

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

constexpr int BM = 128, BK = 64;
// Four epilogue warps per TMEM lane quadrant: the epilogue (TMEM reads,
// residual loads, row stores) is the longer leg of a tile, and with two warps
// per quadrant it ran about twice as long as the tile's MMAs.
constexpr int kParts = 4;
constexpr int kEpiWarps = 4 * kParts;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr size_t kSmemMax = 232448;

template <int BN, int EPI>
struct GemmCfg {
  static constexpr int NI = BN > 256 ? 256 : BN;     // N of one MMA instruction
  static constexpr int NSUB = BN / NI;
  static constexpr int WB = BN < 128 ? BN : 128;     // weight rows per TMA box
  static constexpr int ACC_BUFS = 2 * BN <= 512 ? 2 : 1;
  static constexpr uint32_t TMEM_COLS =
      ACC_BUFS * BN <= 32 ? 32 : ACC_BUFS * BN <= 64 ? 64 : ACC_BUFS * BN <= 128 ? 128
      : ACC_BUFS * BN <= 256 ? 256 : 512;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  // epilogue warps that take part: kParts column parts of 32 or more columns
  static constexpr int P = BN / 32 < kParts ? BN / 32 : kParts;
  // the norm's partial sums and gain only for the norm epilogue
  static constexpr size_t FIXED = 1024 + 256 + kEpiWarps * kStageBytes +
                                  (EPI == TC_NORM ? 2 * kParts * 128 * 4 + BN * 2 : 0);
  // as many stages as fit, at most 8
  static constexpr int STAGES_FIT = (int)((kSmemMax - FIXED) / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
  static constexpr size_t SMEM = FIXED + (size_t)STAGES * STAGE_BYTES;
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(SMEM <= kSmemMax, "shared memory budget");
};

// Epilogue of one 128 x BN tile.  GemmCfg<BN, EPI>::P warps share each TMEM lane
// quadrant; `part` selects which BN / P columns this thread handles.  Stores
// pass through the warp's staging buffer `stg` (row-contiguous global writes).
template <int BN, int EPI>
__device__ __forceinline__ bool epilogue(const TcGemmParams& p, const CUtensorMap* tmD,
                                         uint32_t taddr, int64_t row, bool valid, int n0, int ks,
                                         int g, int part, float* red, int rrow, uint64_t* xbar,
                                         uint32_t& xphase, volatile int* abort_flag, uint32_t stg,
                                         NormPre<BN, 1, GemmCfg<BN, EPI>::P>& pre,
                                         const __nv_bfloat16* sg) {
  constexpr int HB = BN / GemmCfg<BN, EPI>::P;   // columns per thread
  const int c0 = part * HB;
  // the warp's 32 rows start here; with a store map its rows go out as TMA
  // boxes of 32 rows x 32 columns (the first row in use decides)
  const int64_t row0 = row - (threadIdx.x & 31);
  const bool box_live = __any_sync(0xffffffffu, valid);
  if constexpr (EPI == TC_NORM) {
    return norm_epilogue(p.norm, taddr, row, valid, part, red, rrow, xbar, xphase,
                         abort_flag, p.status, stg, pre, sg, p.d_tma ? tmD : nullptr, row0);
  } else if constexpr (EPI == TC_F32) {
    float* prow =
        valid ? p.Dp + ks * p.slice_stride + g * p.d_group_off + row * p.ldp + n0 : nullptr;
#pragma unroll 1
    for (int c = c0; c < c0 + HB; c += 32) {
      float v[32];
      tmem_ld32(taddr + c, v);
      // 32 fp32 = two 64-byte staged row pieces
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          x[j] = make_uint4(__float_as_uint(v[16 * h + 4 * j]), __float_as_uint(v[16 * h + 4 * j + 1]),
                            __float_as_uint(v[16 * h + 4 * j + 2]),
                            __float_as_uint(v[16 * h + 4 * j + 3]));
        stage_store(stg, x, prow ? prow + c + 16 * h : nullptr);
      }
    }
    return true;
  } else {
    int u = 0;
    if (EPI == TC_USERBIAS && valid) u = p.row_user[row];
    __nv_bfloat16* drow = valid ? p.D + row * p.ldd + n0 : nullptr;
    // 32 columns per step (the register budget of 576 threads); the bias
    // loads are issued before the TMEM read
    constexpr int STEP = 32;
#pragma unroll 1
    for (int c = c0; c < c0 + HB; c += STEP) {
      const int n = n0 + c;
      float4 b[STEP / 4];
      if (EPI == TC_USERBIAS && valid) {
        const float4* bp = reinterpret_cast<const float4*>(p.bias + (int64_t)u * p.N + n);
#pragma unroll
        for (int j = 0; j < STEP / 4; ++j) b[j] = __ldg(bp + j);
      }
      float v[STEP];
      tmem_ld32(taddr + c, v);
      if (EPI == TC_USERBIAS && valid) {
#pragma unroll
        for (int j = 0; j < STEP / 4; ++j) {
          v[4 * j] += b[j].x; v[4 * j + 1] += b[j].y; v[4 * j + 2] += b[j].z; v[4 * j + 3] += b[j].w;
        }
      }
#pragma unroll
      for (int h = 0; h < STEP / 32; ++h) {
        uint4 x[4];
        if (EPI == TC_SILU) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[32 * h + i] = silu_approx(v[32 * h + i]);
        }
        pack_bf16x32(&v[32 * h], x);
        if (p.d_tma)
          stage_store_tma(stg, x, tmD, n0 + c + 32 * h, (int32_t)row0, box_live);
        else
          stage_store(stg, x, drow ? drow + c + 32 * h : nullptr);
      }
    }
    return true;
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmD, const TcGemmParams p) {
  using Cfg = GemmCfg<BN, EPI>;
  constexpr int STAGES = Cfg::STAGES, NI = Cfg::NI, NSUB = Cfg::NSUB, ACC_BUFS = Cfg::ACC_BUFS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  // per-warp staging buffers right after the ring (1024-byte aligned: they
  // double as TMA store boxes with the 64-byte swizzle)
  uint8_t* sStage = sB + STAGES * Cfg::B_BYTES;                          // [warp][kStageBytes]
  uint64_t* full = (uint64_t*)(sStage + kEpiWarps * kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + ACC_BUFS;
  uint64_t* drain = tempty + ACC_BUFS;
  uint64_t* xbar = drain + 1;                 // epilogue group barrier (norm exchange)
  uint32_t* tmem_slot = (uint32_t*)(xbar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  // [2 tiles][kParts][128] partial sums of squares (norm epilogue only)
  float* red = (float*)((uint8_t*)full + 256);
  __nv_bfloat16* sG = (__nv_bfloat16*)(red + (EPI == TC_NORM ? 2 * kParts * 128 : 0));   // gain [BN]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.N / BN;
  const int KB = p.K / BK;
  const int kb0 = blockIdx.x % KB;
  const int S = (EPI == TC_F32 && p.k_split > 1) ? p.k_split : 1;   // k-slices (<= KB)
  const int G = (EPI == TC_F32 && p.groups > 1) ? p.groups : 1;      // batch members

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < ACC_BUFS; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], kEpiWarps); }
    mbar_init(drain, 1);
    mbar_init(xbar, 4 * Cfg::P);              // the epilogue warps that take part
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (EPI == TC_NORM) load_gain(p.norm, BN, sG);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier kernels wrote
  pdl_wait();
  const int64_t M = p.M_dev ? *p.M_dev : p.M_host;
  const int64_t mn_tiles = ((M + BM - 1) / BM) * n_tiles;
  const int64_t num_tiles = mn_tiles * G * S;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int64_t tt = t / S;
        const int ks = (int)(t % S);
        const int g = (int)(tt / mn_tiles);
        const int64_t rem = tt % mn_tiles;
        const int mt = (int)(rem / n_tiles), nt = (int)(rem % n_tiles);
        const int a_row = (int)(g * p.a_group_rows) + mt * BM;
        const int w_row = g * p.w_group_rows + nt * BN;
        const int kb_lo = (int)((int64_t)ks * KB / S);
        const int nkb = (int)((int64_t)(ks + 1) * KB / S) - kb_lo;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_sleep(&empty[stage], phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
          // k-blocks in a per-CTA rotated order: the SMs do not all read the
          // same weight lines from L2 at the same moment
          const int kx = (kb_lo + (kb + kb0) % nkb) * BK;
          tma_load_2d(&tmA, &full[stage], sA + stage * Cfg::A_BYTES, kx, a_row);
          // the weight k-block in boxes of at most 128 rows (stacked, they
          // form the same 128-byte-swizzled tile as one box of BN rows)
#pragma unroll
          for (int s2 = 0; s2 < BN / Cfg::WB; ++s2)
            tma_load_2d(&tmB, &full[stage], sB + stage * Cfg::B_BYTES + s2 * Cfg::WB * 128, kx,
                        w_row + s2 * Cfg::WB);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // after an abort the MMA thread may have left stages unread
      if (*abort_flag) drain_ring(full, STAGES, issued, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // A and the weight: both fp16 or both bf16 (the caller's choice)
      const uint32_t IDESC = p.ab_f16 ? idesc_f16(128, NI, false, false)
                                      : idesc_bf16(128, NI, false, false);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait_sleep(&tempty[acc], acc_phase ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_base = tmem + acc * BN;
        const int ks = (int)(t % S);
        const int nkb = (int)((int64_t)(ks + 1) * KB / S) - (int)((int64_t)ks * KB / S);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_sleep(&full[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(a_addr + k * 32, 16, 1024);
#pragma unroll
            for (int s2 = 0; s2 < NSUB; ++s2) {
              const uint64_t bd = sdesc_sw128(b_addr + s2 * NI * 128 + k * 32, 16, 1024);
              umma_bf16(d_base + s2 * NI, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA of this CTA must be complete before TMEM is released
      umma_commit(drain);
      int dummy = 0;
      mbar_wait_sleep(drain, 0, &dummy, p.status);
    }
    __syncwarp();
  } else {
    const int q = warp & 3;                // TMEM lane quadrant this warp may access
    const int part = (warp - 2) >> 2;      // which part of the tile's columns
    const bool active = part < Cfg::P;     // BN = 64: two parts, two warps idle
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    int acc = 0, it = 0;
    uint32_t acc_phase = 0, xphase = 0;
    for (int64_t t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int64_t tt = t / S;
      const int ks = (int)(t % S);
      const int g = (int)(tt / mn_tiles);
      const int64_t rem = tt % mn_tiles;
      const int mt = (int)(rem / n_tiles), nt = (int)(rem % n_tiles);
      const int rr = q * 32 + lane;
      const int64_t row = (int64_t)mt * BM + rr;
      NormPre<BN, 1, Cfg::P> pre;
      if constexpr (EPI == TC_NORM) {
        if (active) norm_prefetch(p.norm, row, row < M, part, pre);
      }
      const bool ok = mbar_wait_sleep(&tfull[acc], acc_phase, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (active &&
          !epilogue<BN, EPI>(p, &tmD, lane_base + acc * BN, row, row < M, nt * BN, ks, g, part,
                             red + (it & 1) * kParts * 128, rr, xbar, xphase, abort_flag,
                             smem_u32(sStage + (warp - 2) * kStageBytes), pre, sG))
        break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1; }
    }
    // the bulk stores must be complete before the CTA ends
    if (p.d_tma) stage_tma_drain();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

template <int BN, int EPI>
cudaError_t launch_cfg(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d,
                       const TcGemmParams& p, int grid, cudaStream_t s) {
  using Cfg = GemmCfg<BN, EPI>;
  static uint64_t attr_devices = 0;   // devices on which the smem limit was raised
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<BN, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  return launch_dependent(tc_gemm_kernel<BN, EPI>, dim3(grid), dim3(kThreads), Cfg::SMEM, s, 1,
                          a, b, d, p);
}

// ---------------------------------------------------------------- SM pairs
// The same GEMM on pairs of SMs for BN = 256: a cluster of two CTAs takes
// 256-row tiles, rank 0 issues cta_group::2 MMAs (M = 256, N = 256), each CTA
// loads its own 128 rows of A and 128 of the 256 weight rows of every k-block
// (the pair's tensor cores read both halves), so that per FLOP a CTA moves
// two thirds of the bytes the one-SM tile moves through L2 and shared
// memory (the one-SM 128 x 256 tile is bound by that traffic).  Each CTA's
// TMEM holds its 128 rows of the accumulator, double-buffered (2 x 256
// columns), and its 16 epilogue warps run the usual epilogues on them.
// Completion of the pair MMAs reaches both CTAs by multicast commit; rank 1's
// "accumulator free" is forwarded to rank 0 by one thread, one remote arrival
// per tile.
template <int EPI>
struct Pair2Cfg {
  static constexpr int BN = 256;
  static constexpr uint32_t A_BYTES = 128 * BK * 2;   // this CTA's 128 rows
  static constexpr uint32_t B_BYTES = 128 * BK * 2;   // this CTA's half of the weight rows
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr size_t FIXED = 1024 + 256 + kEpiWarps * kStageBytes +
                                  (EPI == TC_NORM ? 2 * kParts * 128 * 4 + BN * 2 : 0);
  static constexpr int STAGES_FIT = (int)((kSmemMax - FIXED) / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
  static constexpr size_t SMEM = FIXED + (size_t)STAGES * STAGE_BYTES;
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM <= kSmemMax, "shared memory budget");
};

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_pair2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const TcGemmParams p) {
  using Cfg = Pair2Cfg<EPI>;
  constexpr int BN = 256, STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* sStage = sB + STAGES * Cfg::B_BYTES;                          // [warp][kStageBytes]
  uint64_t* full = (uint64_t*)(sStage + kEpiWarps * kStageBytes);         // [STAGES] rank 0: both CTAs' bytes
  uint64_t* empty = full + STAGES;                                        // [STAGES] both
  uint64_t* tfull = empty + STAGES;                                       // [2] both
  uint64_t* tempty = tfull + 2;                                           // [2] this CTA's epilogue done
  uint64_t* tempty_peer = tempty + 2;                                     // [2] rank 0: rank 1's done
  uint64_t* drain = tempty_peer + 2;
  uint64_t* xbar = drain + 1;                 // epilogue group barrier (norm exchange)
  uint32_t* tmem_slot = (uint32_t*)(xbar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* red = (float*)((uint8_t*)full + 256);
  __nv_bfloat16* sG = (__nv_bfloat16*)(red + (EPI == TC_NORM ? 2 * kParts * 128 : 0));
  static_assert((2 * STAGES + 8) * 8 + 8 <= 256, "barrier area");

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_tiles = p.N / BN;
  const int KB = p.K / BK;
  const int kb0 = pair % KB;

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < STAGES; ++s2) { mbar_init(&full[s2], 1); mbar_init(&empty[s2], 1); }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
      mbar_init(&tempty_peer[a], 1);
    }
    mbar_init(drain, 1);
    mbar_init(xbar, 4 * kParts);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if constexpr (EPI == TC_NORM) load_gain(p.norm, BN, sG);
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier kernels wrote
  pdl_wait();
  const int64_t M = p.M_dev ? *p.M_dev : p.M_host;
  const int64_t num_tiles = ((M + 2 * BM - 1) / (2 * BM)) * n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0;
      bool ok = true;
      for (int64_t t = pair; t < num_tiles && ok; t += n_pairs) {
        const int mt = (int)(t / n_tiles), nt = (int)(t % n_tiles);
        const int32_t a_row = mt * 2 * BM + BM * (int)rank;
        const int32_t w_row = nt * BN + 128 * (int)rank;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_sleep(&empty[stage], phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::STAGE_BYTES);
          const uint32_t full_c = cluster_addr(&full[stage], 0);
          // k-blocks in a per-pair rotated order: the SMs do not all read the
          // same weight lines from L2 at the same moment
          const int kx = ((kb + kb0) % KB) * BK;
          tma_load_2d_pair(&tmA, full_c, sA + stage * Cfg::A_BYTES, kx, a_row);
          tma_load_2d_pair(&tmB, full_c, sB + stage * Cfg::B_BYTES, kx, w_row);
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
      // A and the weight: both fp16 or both bf16 (the caller's choice)
      const uint32_t IDESC = p.ab_f16 ? idesc_f16(2 * BM, BN, false, false)
                                      : idesc_bf16(2 * BM, BN, false, false);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t t = pair; t < num_tiles && ok; t += n_pairs) {
        // both CTAs' epilogues have read this accumulator's previous tile
        if (!mbar_wait_sleep(&tempty[acc], acc_phase ^ 1, abort_flag, p.status) ||
            !mbar_wait_cluster(&tempty_peer[acc], acc_phase ^ 1, abort_flag, p.status))
          break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_sleep(&full[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad0 = sdesc_sw128(smem_u32(sA + stage * Cfg::A_BYTES), 16, 1024);
          const uint64_t bd0 = sdesc_sw128(smem_u32(sB + stage * Cfg::B_BYTES), 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)   // 16 elements of K = 32 bytes per step
            umma_bf16_pair(d, ad0 + (uint64_t)(2 * k), bd0 + (uint64_t)(2 * k), IDESC,
                           (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // every pair MMA must be complete before either CTA releases TMEM
      umma_commit_pair(drain);
      int dummy = 0;
      mbar_wait_sleep(drain, 0, &dummy, p.status);
    } else if (lane == 0) {
      // rank 1: forward this CTA's "accumulator free" to rank 0
      const uint32_t peer_c[2] = {cluster_addr(&tempty_peer[0], 0), cluster_addr(&tempty_peer[1], 0)};
      uint32_t ti = 0;
      for (int64_t t = pair; t < num_tiles; t += n_pairs, ++ti) {
        if (!mbar_wait_sleep(&tempty[ti & 1], (ti >> 1) & 1, abort_flag, p.status)) break;
        mbar_arrive_cluster(peer_c[ti & 1]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                // TMEM lane quadrant this warp may access
    const int part = (warp - 2) >> 2;      // which quarter of the tile's columns
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    int acc = 0, it = 0;
    uint32_t acc_phase = 0, xphase = 0;
    for (int64_t t = pair; t < num_tiles; t += n_pairs, ++it) {
      const int mt = (int)(t / n_tiles), nt = (int)(t % n_tiles);
      const int rr = q * 32 + lane;
      const int64_t row = (int64_t)mt * 2 * BM + BM * (int64_t)rank + rr;
      NormPre<BN, 1, GemmCfg<BN, EPI>::P> pre;
      if constexpr (EPI == TC_NORM) norm_prefetch(p.norm, row, row < M, part, pre);
      const bool ok = mbar_wait_sleep(&tfull[acc], acc_phase, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (!epilogue<BN, EPI>(p, &tmD, lane_base + acc * BN, row, row < M, nt * BN, 0, 0, part,
                             red + (it & 1) * kParts * 128, rr, xbar, xphase, abort_flag,
                             smem_u32(sStage + (warp - 2) * kStageBytes), pre, sG))
        break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    // the bulk stores must be complete before the CTA ends
    if (p.d_tma) stage_tma_drain();
  }
  __syncthreads();
  cluster_sync();          // rank 0's MMAs into both TMEMs are complete
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Pairs of this kernel that can be resident at once.
template <int EPI>
int pair2_max(int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev]) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Pair2Cfg<EPI>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_pair2_kernel<EPI>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  n = std::min(n, num_sms / 2);
  if (dev < 64) cached[dev] = n;
  return n;
}

template <int EPI>
cudaError_t launch_pair2(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d,
                         const TcGemmParams& p, int num_sms, cudaStream_t s) {
  using Cfg = Pair2Cfg<EPI>;
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_pair2_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  const int64_t max_tiles = ((p.M_cap + 2 * BM - 1) / (2 * BM)) * (p.N / 256);
  const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(pair2_max<EPI>(num_sms), max_tiles));
  return launch_dependent(tc_gemm_pair2_kernel<EPI>, dim3(2 * pairs), dim3(kThreads), Cfg::SMEM, s,
                          2, a, b, d, p);
}

template <int EPI>
cudaError_t launch_epi(int BN, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& d,
                       const TcGemmParams& p, int grid, cudaStream_t s) {
  switch (BN) {
    case 64: return launch_cfg<64, EPI>(a, b, d, p, grid, s);
    case 128: return launch_cfg<128, EPI>(a, b, d, p, grid, s);
    case 256: return launch_cfg<256, EPI>(a, b, d, p, grid, s);
    case 512:
      if constexpr (EPI == TC_NORM) return launch_cfg<512, EPI>(a, b, d, p, grid, s);
      else return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool tc_gemm_supported(int BN, int epi, int N, int K) {
  if (K % BK != 0 || K <= 0) return false;
  if (BN != 64 && BN != 128 && BN != 256 && BN != 512) return false;
  if (BN == 512 && epi != TC_NORM) return false;
  if (epi == TC_NORM && N != BN) return false;
  if (epi == TC_F32 && BN > 128) return false;
  return N % BN == 0;
}

cudaError_t launch_tc_gemm(int BN, int epi, const CUtensorMap& a, const CUtensorMap& b,
                           const TcGemmParams& p_in, int num_sms, cudaStream_t s,
                           const CUtensorMap* d) {
  if (!tc_gemm_supported(BN, epi, p_in.N, p_in.K)) return cudaErrorInvalidValue;
  TcGemmParams p = p_in;
  // bulk tensor stores: the plain-store epilogues, and the norm epilogue with
  // one plain output (bf16 dst, or its fp16 residual copy alone)
  p.d_tma = 0;
  if (d && (epi == TC_STORE || epi == TC_USERBIAS || epi == TC_SILU ||
            (epi == TC_NORM && p.norm.mode == NORM_PLAIN && ((p.norm.dst != nullptr) !=
                                                              (p.norm.dst_res != nullptr)))))
    p.d_tma = 1;
  const CUtensorMap& dm = p.d_tma ? *d : a;     // (unused without bulk stores)
  if (epi == TC_F32 &&
      (p.k_split < 1 || p.k_split > p.K / BK || p.groups < 1 || !p.Dp || p.ldp % 4 != 0 ||
       p.d_group_off % 4 != 0 || p.slice_stride % 4 != 0 ||
       (p.groups > 1 && ((p.M_cap > p.a_group_rows) ||
                         (int64_t)p.groups * p.a_group_rows > INT32_MAX ||
                         (int64_t)p.groups * p.w_group_rows > INT32_MAX))))
    return cudaErrorInvalidValue;
  // The FFN up-projection (SiLU, K >= 512) on SM pairs: its one-SM tiles wait
  // on operand traffic.  Measured on the other BN = 256 GEMMs (plain store,
  // per-user bias, norm; K = 256 or N = 256) the pair tiles were no faster or
  // slower, so they keep the one-SM kernel.
  if (BN == 256 && epi == TC_SILU && p.K >= 512) return launch_pair2<TC_SILU>(a, b, dm, p, num_sms, s);
  // grid: one CTA per SM, never more CTAs than the largest possible tile count
  const int64_t max_tiles = ((p.M_cap + BM - 1) / BM) * (p.N / BN) *
                            (epi == TC_F32 ? (int64_t)p.k_split * p.groups : 1);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, max_tiles));
  switch (epi) {
    case TC_STORE: return launch_epi<TC_STORE>(BN, a, b, dm, p, grid, s);
    case TC_USERBIAS: return launch_epi<TC_USERBIAS>(BN, a, b, dm, p, grid, s);
    case TC_SILU: return launch_epi<TC_SILU>(BN, a, b, dm, p, grid, s);
    case TC_NORM: return launch_epi<TC_NORM>(BN, a, b, dm, p, grid, s);
    case TC_F32:
      if (BN == 64) return launch_cfg<64, TC_F32>(a, b, dm, p, grid, s);
      if (BN == 128) return launch_cfg<128, TC_F32>(a, b, dm, p, grid, s);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- tensor maps
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}
}  // namespace

namespace {
// 2-D 16-bit tensor [rows, cols] (row-major, cols contiguous), box of
// box_rows x 64 columns (128 bytes), 128-byte swizzle, zero fill outside.
bool make_tmap_16(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t rows,
                  uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols % 64 != 0 || ((uintptr_t)base & 15) || box_rows > 256) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

bool make_tmap_store16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, bool f16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols % 32 != 0 || ((uintptr_t)base & 15)) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  return make_tmap_16(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rows, cols, box_rows);
}
bool make_tmap_f16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  return make_tmap_16(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, rows, cols, box_rows);
}

}  // namespace llatte
