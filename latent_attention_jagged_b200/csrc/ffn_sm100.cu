// Fused FFN block for sm_100a, d = 256:
//   X = RMSNorm_{g2}(Z + W2 SiLU(W1 Z))       (LLaTTE notes, huaxiaozhuan.com,
//                                              appendix A.2 display; FFN read
//                                              as W2 SiLU(W1 z), hidden 4d)
// with the 4d-wide hidden activation never leaving the SM.
//
// Per 128-row tile: the Z block stays in shared memory; the hidden layer is
// walked in 128-wide chunks j:
//   MMA1(j)  H[j % 2]  = Z W1[j]^T        (TMEM, two 128-column buffers)
//   SiLU(j)  8 epilogue warps: H -> SiLU -> bf16 -> shared memory (A operand)
//   MMA2(j)  OUT      += SiLU(H_j) W2[:, j]^T   (TMEM, 256 columns)
// (each CTA starts at a different chunk and wraps around)
// MMA1(j + 2) is issued right after MMA2(j), so the tensor pipe works on the
// next chunks while the epilogue warps apply SiLU.  After the last chunk the
// same warps run the residual + RMSNorm epilogue on OUT and scatter each row
// into the next layer's history / query rows.
// Roles: warp 0 TMA (Z block, then W1 / W2 k-blocks through a 3-stage ring in
// exactly the order the MMAs consume them), warp 1 TMEM owner + MMA issuer,
// warps 2..9 epilogue (two per TMEM lane quadrant, half the columns each).
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "tc_epilogue.cuh"
#include "tc_ffn.h"

namespace llatte {

using namespace tc;

namespace {

constexpr int D = 256;                      // model width handled here
constexpr int HC = 128;                     // hidden chunk
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int W_STAGES = 3;
constexpr uint32_t Z_BYTES = 128 * D * 2;            // 64 KB: 4 sub-tiles of 128 x 64
constexpr uint32_t HS_BYTES = 128 * HC * 2;          // 32 KB: 2 sub-tiles of 128 x 64
constexpr uint32_t W_STAGE_BYTES = 32768;            // W1: 2 boxes 128 x 64; W2: 1 box 256 x 64
constexpr uint32_t OUT_COL = 0, H_COL = D;           // TMEM columns
constexpr size_t SMEM = 1024 + Z_BYTES + 2 * HS_BYTES + W_STAGES * W_STAGE_BYTES + 256 + D * 2;
static_assert(SMEM <= 232448, "shared memory budget");

__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmW1,
              const __grid_constant__ CUtensorMap tmW2, const FfnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sZ = smem;
  uint8_t* sHs = sZ + Z_BYTES;                         // [2][HS_BYTES]
  uint8_t* sW = sHs + 2 * HS_BYTES;                    // [W_STAGES][W_STAGE_BYTES]
  uint64_t* bars = (uint64_t*)(sW + W_STAGES * W_STAGE_BYTES);
  uint64_t* z_full = bars;
  uint64_t* z_empty = bars + 1;
  uint64_t* w_full = bars + 2;                         // [W_STAGES]
  uint64_t* w_empty = w_full + W_STAGES;               // [W_STAGES]
  uint64_t* h_full = w_empty + W_STAGES;               // [2]
  uint64_t* hs_full = h_full + 2;                      // [2]
  uint64_t* hs_empty = hs_full + 2;                    // [2]
  uint64_t* out_full = hs_empty + 2;
  uint64_t* out_empty = out_full + 1;
  uint64_t* drain = out_empty + 1;
  uint64_t* xbar = drain + 1;                          // epilogue group barrier
  uint32_t* tmem_slot = (uint32_t*)(xbar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  // the residual-norm exchange lives in the first SiLU buffer: while OUT is
  // normalised no MMA reads that buffer and no SiLU chunk is being written
  float* red = (float*)sHs;
  __nv_bfloat16* sG = (__nv_bfloat16*)((uint8_t*)sW + W_STAGES * W_STAGE_BYTES + 256);  // gain [D]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t M = *p.M_dev;
  const int64_t num_tiles = (M + 127) / 128;
  const int NC = p.F / HC;
  // Every CTA walks the hidden chunks in a rotated order, so that the SMs do
  // not all read the same weight lines from L2 at the same moment.
  const int c0 = blockIdx.x % NC;
  auto chunk = [&](int j) { return (c0 + j) % NC; };

  if (threadIdx.x == 0) {
    mbar_init(z_full, 1);
    mbar_init(z_empty, 1);
    for (int s = 0; s < W_STAGES; ++s) { mbar_init(&w_full[s], 1); mbar_init(&w_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&h_full[b], 1);
      mbar_init(&hs_full[b], kEpiWarps);
      mbar_init(&hs_empty[b], 1);
    }
    mbar_init(out_full, 1);
    mbar_init(out_empty, kEpiWarps);
    mbar_init(drain, 1);
    mbar_init(xbar, kEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmZ);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  load_gain(p.norm, D, sG);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t w = 0, ti = 0;
      bool ok = true;
      auto next_stage = [&](uint32_t bytes) -> uint8_t* {
        const int st = w % W_STAGES;
        if (!mbar_wait(&w_empty[st], ((w / W_STAGES) & 1) ^ 1, abort_flag, p.status)) return nullptr;
        mbar_arrive_expect_tx(&w_full[st], bytes);
        return sW + st * W_STAGE_BYTES;
      };
      auto load_w1 = [&](int j) -> bool {     // W1 rows j*HC .. +128, all D columns
        for (int s2 = 0; s2 < 2; ++s2) {
          uint8_t* dst = next_stage(W_STAGE_BYTES);
          if (!dst) return false;
          const int st = w % W_STAGES;
          tma_load_2d(&tmW1, &w_full[st], dst, 128 * s2, j * HC);
          tma_load_2d(&tmW1, &w_full[st], dst + 16384, 128 * s2 + 64, j * HC);
          ++w;
        }
        return true;
      };
      auto load_w2 = [&](int j) -> bool {     // W2 all D rows, columns j*HC .. +128
        for (int s2 = 0; s2 < 2; ++s2) {
          uint8_t* dst = next_stage(W_STAGE_BYTES);
          if (!dst) return false;
          const int st = w % W_STAGES;
          tma_load_2d(&tmW2, &w_full[st], dst, j * HC + 64 * s2, 0);
          ++w;
        }
        return true;
      };
      for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++ti) {
        if (!mbar_wait(z_empty, (ti & 1) ^ 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(z_full, Z_BYTES);
        for (int s = 0; s < D / 64; ++s) tma_load_2d(&tmZ, z_full, sZ + s * 16384, 64 * s, (int)(t * 128));
        ok = load_w1(chunk(0)) && (NC < 2 || load_w1(chunk(1)));
        for (int j = 0; j < NC && ok; ++j) {
          ok = load_w2(chunk(j)) && (j + 2 >= NC || load_w1(chunk(j + 2)));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC1 = idesc_bf16(128, HC, false, false);
      constexpr uint32_t IDESC2 = idesc_bf16(128, D, false, false);
      const uint32_t z_addr = smem_u32(sZ);
      uint32_t w = 0, ti = 0, gc = 0;
      bool ok = true;
      auto mma1 = [&](int j, uint32_t gcj) -> bool {   // H[gcj&1] = Z W1[chunk(j)]^T
        const uint32_t d = tmem + H_COL + (gcj & 1) * HC;
        for (int s2 = 0; s2 < 2; ++s2) {
          const int st = w % W_STAGES;
          if (!mbar_wait(&w_full[st], (w / W_STAGES) & 1, abort_flag, p.status)) return false;
          tc_fence_after();
          const uint32_t wb = smem_u32(sW + st * W_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t ad = sdesc_sw128(z_addr + (2 * s2 + (k >> 2)) * 16384 + (k & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(wb + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
            umma_bf16(d, ad, bd, IDESC1, (s2 | k) != 0 ? 1u : 0u);
          }
          umma_commit(&w_empty[st]);
          ++w;
        }
        umma_commit(&h_full[gcj & 1]);
        if (j == NC - 1) umma_commit(z_empty);
        return true;
      };
      auto mma2 = [&](int j, uint32_t gcj) -> bool {   // OUT += SiLU(H_j) W2[:, chunk(j)]^T
        if (!mbar_wait(&hs_full[gcj & 1], (gcj >> 1) & 1, abort_flag, p.status)) return false;
        if (j == 0 && !mbar_wait(out_empty, (ti & 1) ^ 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t hs = smem_u32(sHs + (gcj & 1) * HS_BYTES);
        for (int s2 = 0; s2 < 2; ++s2) {
          const int st = w % W_STAGES;
          if (!mbar_wait(&w_full[st], (w / W_STAGES) & 1, abort_flag, p.status)) return false;
          tc_fence_after();
          const uint32_t wb = smem_u32(sW + st * W_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_sw128(hs + s2 * 16384 + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(wb + k * 32, 16, 1024);
            umma_bf16(tmem + OUT_COL, ad, bd, IDESC2, (j | s2 | k) != 0 ? 1u : 0u);
          }
          umma_commit(&w_empty[st]);
          ++w;
        }
        umma_commit(&hs_empty[gcj & 1]);
        if (j == NC - 1) umma_commit(out_full);
        return true;
      };
      for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++ti) {
        if (!mbar_wait(z_full, ti & 1, abort_flag, p.status)) break;
        ok = mma1(0, gc) && (NC < 2 || mma1(1, gc + 1));
        for (int j = 0; j < NC && ok; ++j) {
          ok = mma2(j, gc + j) && (j + 2 >= NC || mma1(j + 2, gc + j + 2));
        }
        gc += NC;
      }
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, &dummy, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int rr = q * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t ti = 0, gc = 0, xphase = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++ti) {
      for (int j = 0; j < NC; ++j, ++gc) {
        bool w1 = mbar_wait(&h_full[gc & 1], (gc >> 1) & 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
        tc_fence_after();
        float v[2][32];
        tmem_ld32(lane_base + H_COL + (gc & 1) * HC + half * 64, v[0]);
        tmem_ld32(lane_base + H_COL + (gc & 1) * HC + half * 64 + 32, v[1]);
        bool w2 = mbar_wait(&hs_empty[gc & 1], ((gc >> 1) & 1) ^ 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
        // SiLU -> bf16 -> 128-byte-swizzled K-major tile (sub-tile = half)
        const uint32_t base = smem_u32(sHs + (gc & 1) * HS_BYTES + half * 16384) + rr * 128;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const float* x = &v[cc >> 2][(cc & 3) * 8];
          uint4 o = make_uint4(pack_bf16(silu_approx(x[0]), silu_approx(x[1])),
                               pack_bf16(silu_approx(x[2]), silu_approx(x[3])),
                               pack_bf16(silu_approx(x[4]), silu_approx(x[5])),
                               pack_bf16(silu_approx(x[6]), silu_approx(x[7])));
          st_shared_v4(base + ((cc ^ (rr & 7)) << 4), o);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&hs_full[gc & 1]);
      }
      if (!ok) break;
      const int64_t row = t * 128 + rr;
      NormPre<D, 2> pre;   // two chunks ahead: the register budget is tight here
      norm_prefetch(p.norm, row, row < M, half, pre);
      bool w3 = mbar_wait(out_full, ti & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w3)) break;
      tc_fence_after();
      // staging buffers: in the first hidden tile, after `red` (both hidden
      // tiles are idle while the output epilogue runs; the group barrier
      // below keeps the next SiLU chunk out until every warp is done)
      if (!norm_epilogue(p.norm, lane_base + OUT_COL, row, row < M, half, red, rr, xbar,
                            xphase, abort_flag, p.status,
                            smem_u32(sHs) + 1024 + (warp - 2) * kStageBytes, pre, sG))
        break;
      // every partner has read `red` before a SiLU chunk reuses that memory
      if (!group_sync(xbar, xphase, abort_flag, p.status)) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_empty);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool ffn_tc_supported(int d, int f) { return d == D && f % HC == 0 && f >= HC; }

cudaError_t launch_ffn_tc(const CUtensorMap& z, const CUtensorMap& w1, const CUtensorMap& w2,
                          const FfnTcParams& p, int num_sms, cudaStream_t s) {
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(ffn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  const int64_t max_tiles = (p.M_cap + 127) / 128;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms, max_tiles));
  ffn_tc_kernel<<<grid, kThreads, SMEM, s>>>(z, w1, w2, p);
  return cudaGetLastError();
}

}  // namespace llatte
