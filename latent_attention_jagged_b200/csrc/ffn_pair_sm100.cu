// Fused FFN block for sm_100a, d = 256, on pairs of SMs:
//   X = RMSNorm_{g2}(Z + W2 SiLU(W1 Z))       (LLaTTE notes, huaxiaozhuan.com,
//                                              appendix A.2 display; FFN read
//                                              as W2 SiLU(W1 z), hidden 4d)
// with the 4d-wide hidden activation never leaving the SMs.
//
// A cluster of two CTAs (one per SM) takes 256-row tiles: CTA rank r owns
// rows [256 t + 128 r, +128) of tile t.  The tensor cores of the pair work as
// one (cta_group::2): rank 0 issues every MMA with M = 256; each CTA holds its
// own 128 rows of the A operand and HALF of the B operand (the weight chunk),
// so that every weight byte crosses L2 and shared memory once per 256 rows
// instead of once per 128.  Each CTA's TMEM holds its rows of the
// accumulators, and the hidden activation never touches shared memory:
//   MMA1(j)  H[j % 2]  = Z W1[j]^T        (two 128-column TMEM buffers)
//   SiLU(j)  8 warps per CTA: H -> SiLU -> bf16, written back over H in TMEM
//   MMA2(j)  OUT      += SiLU(H_j) W2[:, j]^T   (A read from TMEM; 256 columns)
// walking the hidden layer in 128-wide chunks j (each pair starts at a
// different chunk and wraps around); MMA1(j + 2) is issued right after
// MMA2(j) (the tensor pipe runs one thread's MMAs in issue order, so MMA1(j + 2)
// overwrites H[j % 2] only after MMA2(j) has read it).  After the last chunk
// the same warps run the residual + RMSNorm
// epilogue on OUT and scatter each row into the next layer's history / query
// rows.
// Roles per CTA: warp 0 TMA (Z block, then this CTA's halves of the W1 / W2
// chunks through a 3-stage ring, in the order the MMAs consume them; the
// bytes of both CTAs are counted on rank 0's barriers), warp 1 TMEM owner
// (in rank 0 also the MMA issuer), warps 2..9 SiLU and the OUT copy, warps
// 10..17 the row epilogue (16 rows each: with four warps the row epilogue set
// the pace of the whole tile).  Completion of the pair MMAs is signalled to
// both CTAs at once (multicast commit); the SiLU and OUT-copy warps of both
// CTAs arrive directly on rank 0's barriers (rank 1's with remote arrivals),
// so the issuer waits on one barrier per chunk.
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
constexpr int kSiluWarps = 8;               // two per TMEM lane quadrant
constexpr int kRowWarps = 8;                // row epilogue
constexpr int kRowsPerWarp = 128 / kRowWarps;
constexpr int kRowWarp0 = 2 + kSiluWarps;
constexpr int kThreads = 32 * (2 + kSiluWarps + kRowWarps);
constexpr int W_STAGES = 3;
constexpr uint32_t Z_BYTES = 128 * D * 2;            // 64 KB: 4 sub-tiles of 128 x 64
constexpr uint32_t V_BYTES = 128 * D * 2;            // OUT as fp16, [128][D], 16-byte chunks swizzled
// one stage = this CTA's half of a weight chunk:
//   W1 rows [j HC + 64 r, +64) x all D columns: 4 boxes of 64 x 64 (8 KB)
//   W2 rows [128 r, +128) x columns [j HC, +128): 2 boxes of 128 x 64 (16 KB)
constexpr uint32_t W_STAGE_BYTES = 32768;
constexpr uint32_t OUT_COL = 0, H_COL = D;           // TMEM columns
constexpr size_t SMEM = 1024 + Z_BYTES + W_STAGES * W_STAGE_BYTES + V_BYTES + 256 + D * 2;
static_assert(SMEM <= 232448, "shared memory budget");

__global__ void __launch_bounds__(kThreads, 1)
ffn_pair_kernel(const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmW1,
                const __grid_constant__ CUtensorMap tmW2, const FfnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sZ = smem;
  uint8_t* sW = sZ + Z_BYTES;                          // [W_STAGES][W_STAGE_BYTES]
  uint8_t* sV = sW + W_STAGES * W_STAGE_BYTES;         // OUT rows, fp16
  uint64_t* bars = (uint64_t*)(sV + V_BYTES);
  uint64_t* z_full = bars;                             // rank 0: both Z halves in
  uint64_t* z_empty = bars + 1;                        // both: last MMA1 of the tile done
  uint64_t* w_full = bars + 2;                         // [W_STAGES] rank 0: both halves in
  uint64_t* w_empty = w_full + W_STAGES;               // [W_STAGES] both
  uint64_t* h_full = w_empty + W_STAGES;               // [2] both
  uint64_t* hs_done = h_full + 2;                      // [2] rank 0: both CTAs' SiLU warps done
  uint64_t* out_full = hs_done + 2;                    // both
  uint64_t* out_free = out_full + 1;                   // rank 0: both CTAs' OUT copies done
  uint64_t* v_full = out_free + 1;                     // both: OUT copied to sV
  uint64_t* v_free = v_full + 1;                       // both: row epilogue done with sV
  uint64_t* drain = v_free + 1;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  __nv_bfloat16* sG = (__nv_bfloat16*)((uint8_t*)bars + 256);   // gain [D]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int NC = p.F / HC;
  // Every pair walks the hidden chunks in a rotated order, so that the SMs
  // do not all read the same weight lines from L2 at the same moment.
  const int c0 = pair % NC;
  auto chunk = [&](int j) { return (c0 + j) % NC; };

  if (threadIdx.x == 0) {
    mbar_init(z_full, 1);
    mbar_init(z_empty, 1);
    for (int s = 0; s < W_STAGES; ++s) { mbar_init(&w_full[s], 1); mbar_init(&w_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&h_full[b], 1);
      mbar_init(&hs_done[b], 2 * kSiluWarps);
    }
    mbar_init(out_full, 1);
    mbar_init(out_free, 2 * kSiluWarps);
    mbar_init(v_full, kSiluWarps);
    mbar_init(v_free, kRowWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmZ);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (p.norm.mode != NORM_NONE)
    for (int i = threadIdx.x; i < D / 8; i += blockDim.x)
      reinterpret_cast<uint4*>(sG)[i] = __ldg(reinterpret_cast<const uint4*>(p.norm.g) + i);
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier kernels wrote
  pdl_wait();
  const int64_t M = *p.M_dev;
  const int64_t num_tiles = (M + 255) / 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const bool lead = rank == 0;
      const uint32_t z_full_c = cluster_addr(z_full, 0);
      uint32_t w = 0, ti = 0;
      bool ok = true;
      // next ring stage; rank 0 announces the bytes of both CTAs
      auto next_stage = [&](uint32_t& bar_c) -> uint8_t* {
        const int st = w % W_STAGES;
        if (!mbar_wait(&w_empty[st], ((w / W_STAGES) & 1) ^ 1, abort_flag, p.status)) return nullptr;
        if (lead) mbar_arrive_expect_tx(&w_full[st], 2 * W_STAGE_BYTES);
        bar_c = cluster_addr(&w_full[st], 0);
        return sW + st * W_STAGE_BYTES;
      };
      auto load_w1 = [&](int j) -> bool {     // W1 rows j*HC + 64 rank .. +64, all D columns
        uint32_t bar_c;
        uint8_t* dst = next_stage(bar_c);
        if (!dst) return false;
        for (int b = 0; b < 4; ++b)
          tma_load_2d_pair(&tmW1, bar_c, dst + b * 8192, 64 * b, j * HC + 64 * (int)rank);
        ++w;
        return true;
      };
      auto load_w2 = [&](int j) -> bool {     // W2 rows 128 rank .. +128, columns j*HC .. +128
        uint32_t bar_c;
        uint8_t* dst = next_stage(bar_c);
        if (!dst) return false;
        for (int b = 0; b < 2; ++b)
          tma_load_2d_pair(&tmW2, bar_c, dst + b * 16384, j * HC + 64 * b, 128 * (int)rank);
        ++w;
        return true;
      };
      for (int64_t t = pair; t < num_tiles && ok; t += n_pairs, ++ti) {
        if (!mbar_wait(z_empty, (ti & 1) ^ 1, abort_flag, p.status)) break;
        if (lead) mbar_arrive_expect_tx(z_full, 2 * Z_BYTES);
        const int32_t zrow = (int32_t)(t * 256 + 128 * rank);
        for (int s = 0; s < D / 64; ++s) tma_load_2d_pair(&tmZ, z_full_c, sZ + s * 16384, 64 * s, zrow);
        ok = load_w1(chunk(0)) && (NC < 2 || load_w1(chunk(1)));
        for (int j = 0; j < NC && ok; ++j) {
          ok = load_w2(chunk(j)) && (j + 2 >= NC || load_w1(chunk(j + 2)));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (lane == 0 && rank == 0) {
      // Z W1^T: both operands fp16 or both bf16 (the caller's choice)
      const uint32_t IDESC1 = p.z_f16 ? idesc_f16(256, HC, false, false)
                                      : idesc_bf16(256, HC, false, false);
      constexpr uint32_t IDESC2 = idesc_bf16(256, D, false, false);
      // shared-memory descriptors: the start-address field is (address >> 4),
      // so a k-step or stage offset is a constant added to a base descriptor
      // (every address here is below 256 KB: no carry out of the field)
      const uint64_t z_desc = sdesc_sw128(smem_u32(sZ), 16, 1024);
      const uint64_t w_desc = sdesc_sw128(smem_u32(sW), 16, 1024);
      uint32_t w = 0, ti = 0, gc = 0;
      bool ok = true;
      auto mma1 = [&](int j, uint32_t gcj) -> bool {   // H[gcj&1] = Z W1[chunk(j)]^T
        const uint32_t d = tmem + H_COL + (gcj & 1) * HC;
        const int st = w % W_STAGES;
        if (!mbar_wait(&w_full[st], (w / W_STAGES) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint64_t wd = w_desc + (uint64_t)(st * (W_STAGE_BYTES >> 4));
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_bf16_pair(d, z_desc + (uint64_t)((k >> 2) * (16384 >> 4) + (k & 3) * 2),
                         wd + (uint64_t)((k >> 2) * (8192 >> 4) + (k & 3) * 2), IDESC1, k != 0 ? 1u : 0u);
        umma_commit_pair(&w_empty[st]);
        ++w;
        umma_commit_pair(&h_full[gcj & 1]);
        if (j == NC - 1) umma_commit_pair(z_empty);
        return true;
      };
      auto mma2 = [&](int j, uint32_t gcj) -> bool {   // OUT += SiLU(H_j) W2[:, chunk(j)]^T
        // SiLU(H_j) of both CTAs in TMEM; for the first chunk of a tile also
        // both CTAs' OUT copies done
        if (!mbar_wait_cluster(&hs_done[gcj & 1], (gcj >> 1) & 1, abort_flag, p.status)) return false;
        if (j == 0 && !mbar_wait_cluster(out_free, (ti & 1) ^ 1, abort_flag, p.status)) return false;
        const int st = w % W_STAGES;
        if (!mbar_wait(&w_full[st], (w / W_STAGES) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        // A = SiLU(H_j) as bf16 pairs: hidden columns [64 h, 64 h + 64) were
        // packed into the first 32 columns of that half of the buffer
        const uint32_t ha = tmem + H_COL + (gcj & 1) * HC;
        const uint64_t wd = w_desc + (uint64_t)(st * (W_STAGE_BYTES >> 4));
#pragma unroll
        for (int k = 0; k < HC / 16; ++k)
          umma_bf16_pair_ts(tmem + OUT_COL, ha + (k >> 2) * 64 + (k & 3) * 8,
                            wd + (uint64_t)((k >> 2) * (16384 >> 4) + (k & 3) * 2), IDESC2,
                            (j | k) != 0 ? 1u : 0u);
        umma_commit_pair(&w_empty[st]);
        ++w;
        if (j == NC - 1) umma_commit_pair(out_full);
        return true;
      };
      for (int64_t t = pair; t < num_tiles && ok; t += n_pairs, ++ti) {
        if (!mbar_wait(z_full, ti & 1, abort_flag, p.status)) break;
        ok = mma1(0, gc) && (NC < 2 || mma1(1, gc + 1));
        for (int j = 0; j < NC && ok; ++j) {
          ok = mma2(j, gc + j) && (j + 2 >= NC || mma1(j + 2, gc + j + 2));
        }
        gc += NC;
      }
      // every pair MMA must be complete before either CTA releases TMEM
      umma_commit_pair(drain);
      int dummy = 0;
      mbar_wait(drain, 0, &dummy, p.status);
    }
    __syncwarp();
  } else if (warp < kRowWarp0) {
    // ------------------------------------------------------------ SiLU + OUT copy
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int rr = q * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t vrow = smem_u32(sV) + rr * (D * 2);
    uint32_t ti = 0, gc = 0;
    bool ok = true;
    for (int64_t t = pair; t < num_tiles && ok; t += n_pairs, ++ti) {
      for (int j = 0; j < NC; ++j, ++gc) {
        bool w1 = mbar_wait(&h_full[gc & 1], (gc >> 1) & 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
        tc_fence_after();
        // this warp's 64 hidden columns: SiLU -> bf16 pairs, written over the
        // first 32 columns of its half of the buffer, 32 columns at a time
        // (pass h = 1 reads columns 32..63 and writes packed columns 16..31,
        // which pass h = 0 has already read)
        const uint32_t hcol = lane_base + H_COL + (gc & 1) * HC + half * 64;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float v[32];
          tmem_ld32(hcol + 32 * h, v);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(silu_approx(v[2 * i]), silu_approx(v[2 * i + 1]));
          tmem_st16u(hcol + 16 * h, pk);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {       // on rank 0's barrier (cluster release for rank 1's TMEM writes)
          if (rank == 0) mbar_arrive(&hs_done[gc & 1]);
          else mbar_arrive_cluster(cluster_addr(&hs_done[gc & 1], 0));
        }
      }
      if (!ok) break;
      // OUT (this warp's 128 columns of its row) -> fp16 -> sV, which frees
      // the accumulator for the next tile; 16-byte chunk c of row r sits at
      // chunk c ^ (r % 32)
      bool w3 = mbar_wait(out_full, ti & 1, abort_flag, p.status);
      bool w4 = mbar_wait(v_free, (ti & 1) ^ 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w3 && w4)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = half * 128; c < half * 128 + 128; c += 32) {
        float o[32];
        tmem_ld32(lane_base + OUT_COL + c, o);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float* x = &o[8 * k];
          const uint4 w = make_uint4(pack_f16(x[0], x[1]), pack_f16(x[2], x[3]),
                                     pack_f16(x[4], x[5]), pack_f16(x[6], x[7]));
          const int chunk16 = (c >> 3) + k;
          st_shared_v4(vrow + ((chunk16 ^ (rr & 31)) << 4), w);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(out_free);     // OUT may be overwritten
        else mbar_arrive_cluster(cluster_addr(out_free, 0));
        mbar_arrive(v_full);        // the row warps may read sV
      }
    }
  } else {
    // ------------------------------------------------------------ row epilogue
    // Z + OUT, RMSNorm, gain, scatter into the next layer's rows (LLaTTE
    // notes, huaxiaozhuan.com, appendix A.2 display).  Warp w takes rows
    // kRowsPerWarp (w - kRowWarp0) .. + kRowsPerWarp of the CTA's 128; a row
    // is one warp instruction wide: lane l owns columns [8 l, 8 l + 8).
    const NormArgs& a = p.norm;
    const int r0 = (warp - kRowWarp0) * kRowsPerWarp;
    float g8[8];
    {
      const uint4 gw = reinterpret_cast<const uint4*>(sG)[lane];
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(g2[k]);
        g8[2 * k] = f.x;
        g8[2 * k + 1] = f.y;
      }
    }
    uint32_t ti = 0;
    constexpr int RB = kRowsPerWarp < 8 ? kRowsPerWarp : 8;   // rows whose residual is in flight
    for (int64_t t = pair; t < num_tiles; t += n_pairs, ++ti) {
      const int64_t row_base = t * 256 + 128 * rank;
      if (a.mode == NORM_NONE) {
        // the block's output rows as they are (the action tokenizer's MLP):
        // OUT (fp16 in sV) -> bf16 row of dst, one row per warp instruction
        bool w = mbar_wait(v_full, ti & 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) break;
#pragma unroll 4
        for (int i = 0; i < kRowsPerWarp; ++i) {
          const int r = r0 + i;
          const int64_t row = row_base + r;
          if (row >= M) break;                          // warp-uniform
          const uint4 vw = ld_shared_v4(smem_u32(sV) + r * (D * 2) + ((lane ^ (r & 31)) << 4));
          const __half2* h2 = reinterpret_cast<const __half2*>(&vw);
          uint32_t o[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(h2[k]);
            o[k] = pack_bf16(f.x, f.y);
          }
          *reinterpret_cast<uint4*>((__nv_bfloat16*)a.dst + row * D + 8 * lane) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(v_free);
        continue;
      }
      // destinations of the warp's rows, lane l -> row r0 + l, found before
      // the data is ready (one round of dependent loads for all rows): the
      // next layer's history row, its query row, the final row (-1: none)
      int64_t h_dst = -1, q_dst = -1, f_dst = -1;
      {
        const int64_t row = row_base + r0 + lane;
        if (lane < kRowsPerWarp && row < M) {
          const int u = a.row_user[row];
          const int64_t jr = row - a.qoff_l[u];
          const int32_t nl = a.n_l[u];
          if (a.last) {
            if (a.zraw) {
              if (jr >= nl) h_dst = (int64_t)u * a.n_q + (jr - nl);   // summary input row
            } else if (a.final_rows) {
              f_dst = row;
            } else if (jr >= nl) {
              f_dst = (int64_t)u * a.n_q + (jr - nl);
            }
          } else {
            const int32_t nn = a.n_n[u];
            if (jr < nl) {
              h_dst = a.hoff_n[u] + jr;
              if (jr >= nl - nn) q_dst = a.qoff_n[u] + jr - (nl - nn);
            } else {
              q_dst = a.qoff_n[u] + nn + (jr - nl);
            }
          }
        }
      }
      float* const f_base = a.final_rows ? a.final_rows : a.out;
      __nv_bfloat16* const h_base = (__nv_bfloat16*)(a.last ? a.zraw : a.Xh_n);
      bool w = mbar_wait(v_full, ti & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) break;
#pragma unroll 1
      for (int rb = 0; rb < kRowsPerWarp; rb += RB) {
        uint4 res[RB];
#pragma unroll
        for (int i = 0; i < RB; ++i) {
          const int64_t row = row_base + r0 + rb + i;
          res[i] = row < M ? __ldg(reinterpret_cast<const uint4*>(
                                 (const char*)a.resid + (row * D + 8 * lane) * 2))
                           : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < RB; ++i) {
          const int r = r0 + rb + i;
          const int64_t row = row_base + r;
          const int64_t hd = __shfl_sync(0xffffffffu, h_dst, rb + i);
          const int64_t qd = __shfl_sync(0xffffffffu, q_dst, rb + i);
          const int64_t fd = __shfl_sync(0xffffffffu, f_dst, rb + i);
          if (row >= M) continue;                         // warp-uniform
          const uint4 vw = ld_shared_v4(smem_u32(sV) + r * (D * 2) + ((lane ^ (r & 31)) << 4));
          float x[8];
          {
            const __half2* h2 = reinterpret_cast<const __half2*>(&vw);
            const uint4 rw = res[i];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = __half22float2(h2[k]);
              float2 rf;
              if (a.resid_kind == RES_F16) rf = __half22float2(reinterpret_cast<const __half2*>(&rw)[k]);
              else rf = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&rw)[k]);
              x[2 * k] = f.x + rf.x;
              x[2 * k + 1] = f.y + rf.y;
            }
          }
          float ss = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) ss = fmaf(x[k], x[k], ss);
          ss = warp_sum(ss);
          const float inv = rsqrtf(ss / (float)D + a.eps);
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] *= inv * g8[k];
          const uint4 wb = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                      pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
          if (hd >= 0) *reinterpret_cast<uint4*>(h_base + hd * D + 8 * lane) = wb;
          if (qd >= 0) {
            if (a.Xq_n) *reinterpret_cast<uint4*>((__nv_bfloat16*)a.Xq_n + qd * D + 8 * lane) = wb;
            if (a.Xq_res_n)
              *reinterpret_cast<uint4*>((__half*)a.Xq_res_n + qd * D + 8 * lane) =
                  make_uint4(pack_f16(x[0], x[1]), pack_f16(x[2], x[3]), pack_f16(x[4], x[5]),
                             pack_f16(x[6], x[7]));
          }
          if (fd >= 0) {
            float4* fp = reinterpret_cast<float4*>(f_base + fd * D + 8 * lane);
            fp[0] = make_float4(x[0], x[1], x[2], x[3]);
            fp[1] = make_float4(x[4], x[5], x[6], x[7]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(v_free);
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
  if (cudaOccupancyMaxActiveClusters(&n, ffn_pair_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  n = std::min(n, num_sms / 2);
  if (dev < 64) cached[dev] = n;
  return n;
}

}  // namespace

bool ffn_tc_supported(int d, int f) { return d == D && f % HC == 0 && f >= HC; }

cudaError_t launch_ffn_pair(const CUtensorMap& z, const CUtensorMap& w1h, const CUtensorMap& w2h,
                            const FfnTcParams& p, int num_sms, cudaStream_t s) {
  // the row epilogue implements the scatter into the next layer's rows and the
  // plain store of the tokenizer's MLP
  if ((p.norm.mode != NORM_SCATTER && p.norm.mode != NORM_NONE) || p.F % HC != 0 ||
      (p.norm.mode == NORM_NONE && (!p.norm.dst || ((uintptr_t)p.norm.dst & 15))))
    return cudaErrorInvalidValue;
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(ffn_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  const int64_t max_tiles = (p.M_cap + 255) / 256;
  const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(max_pairs(num_sms), max_tiles));
  return launch_dependent(ffn_pair_kernel, dim3(2 * pairs), dim3(kThreads), SMEM, s, 2, z, w1h, w2h, p);
}

}  // namespace llatte
