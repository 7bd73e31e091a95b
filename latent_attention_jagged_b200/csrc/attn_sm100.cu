// Fused latent attention for sm_100a (MLA as multi-query attention in the
// rank-r latent space, LLaTTE notes, huaxiaozhuan.com, appendix A.3; target-
// aware causal / candidate masking of appendix A.2 and the daiwk.github.io
// "core formula").
//
// One work item = one user u and a block of 128 (query row, head) pairs of
// that user (q~ rows of [sum q * h, r], heads interleaved, so all heads of a
// query row share its mask).  Keys and values are the same latent rows c_kv
// of the user's current history: S = Q~ C^T and O~ = softmax(S) C both read
// one shared-memory copy of each C tile (K-major for S, MN-major for P V).
//
// Roles (448 threads, one CTA per SM, persistent over the sorted work list):
//   warp 0       TMA: the Q~ block once per item, 128-key C tiles into a ring
//                (4 stages, 2 for r = 256)
//   warp 1       TMEM owner; lane 0 issues S(kt+1) = Q~ C_{kt+1}^T before
//                O += P(kt) C_kt, so the tensor pipe works while the softmax
//                warps turn S(kt) into P(kt)
//   warps 2..9   softmax, two warps per TMEM lane quadrant, each taking half
//                of the tile's keys for the quadrant's 32 pairs (one pair per
//                thread): masking (history row at position p sees keys
//                t <= p; a query token sees every key t < T), row max (the two
//                halves meet in shared memory behind a bounded pair barrier),
//                2^(s - m) in fp32, P written back over S in TMEM as bf16,
//                lazy rescaling of O in TMEM (only when the running max grows
//                by more than 2^8)
//   warps 10..13 epilogue: O / l from TMEM to HBM, so the softmax warps move
//                on to the next item at once
// (MLA in its per-head form runs in its own kernel, attn_heads_sm100.cu.)
// TMEM: O (double-buffered across items when 2 r + 2 KEYS <= 512 columns),
// then S double-buffered across key tiles; P(kt) overwrites S(kt) and the
// P V product reads it from TMEM.  The MMAs of one thread run in issue order,
// so S(kt + 2) (issued after P(kt) V) cannot overwrite P(kt) early.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_attn.h"
#include "tc_common.cuh"
#include "tc_drain.cuh"
#include "tc_epilogue.cuh"

namespace llatte {

using namespace tc;

namespace {

constexpr int kSplit = 2;                          // softmax warps per lane quadrant
constexpr int kSoftWarps = 4 * kSplit;
constexpr int kEpiWarps = 4;
constexpr int kEpiWarp0 = 2 + kSoftWarps;
constexpr int kThreads = 32 * (2 + kSoftWarps + kEpiWarps);

template <int R>
struct AttnCfg {
  // 128 keys per tile for every rank: the S MMA then has N = 128 (an N = 64
  // MMA takes about 54 cycles instead of 32 on this part)
  static constexpr int KEYS = 128;
  static constexpr int KP = KEYS / kSplit;             // keys per softmax warp
  static constexpr int RSUB = R / 64;                  // 64-wide latent sub-tiles
  static constexpr int OBUF = (2 * R + 2 * KEYS <= 512) ? 2 : 1;
  static constexpr int QBUF = R <= 128 ? 2 : 1;          // query blocks in flight
  static constexpr int KV_STAGES = R >= 256 ? 2 : 4;   // 64 KB or 32 KB per C tile
  static constexpr uint32_t Q_BYTES = 128 * R * 2;
  static constexpr uint32_t KV_BYTES = KEYS * R * 2;    // one latent tile (K = V)
  static constexpr uint32_t KV_SUB_BYTES = KEYS * 128;  // one 64-wide sub-tile of a C tile
  static constexpr uint32_t S_COL = OBUF * R;           // S buffers after O
  static constexpr uint32_t BAR_BYTES = 256;
  static constexpr uint32_t L_BYTES = 2 * 128 * 4;      // row sums handed to the epilogue
  static constexpr uint32_t MX_BYTES = 2 * kSplit * 128 * 4;   // partial row maxima
  static constexpr size_t SMEM = 1024 + QBUF * Q_BYTES + (size_t)KV_STAGES * KV_BYTES +
                                 BAR_BYTES + L_BYTES + MX_BYTES + kEpiWarps * kStageBytes;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(OBUF * R + 2 * KEYS <= 512, "TMEM budget");
  static_assert(KP == 64, "softmax chunk");
};

// TMEM column (relative to the S buffer) of the packed bf16 P for keys
// [16 kk, 16 kk + 16): each softmax warp packs its KP keys into the first
// KP / 2 columns of its own half of the buffer.
template <int KP>
__device__ __forceinline__ uint32_t p_col(int kk) {
  const int key = 16 * kk;
  return (uint32_t)((key / KP) * KP + (key % KP) / 2);
}

struct Item {
  int u, b;
  int32_t T, n, q;
  int nk;         // key tiles (0: no key at all)
  int64_t hoff, qoff;
};

// The items of one CTA (idx = blockIdx.x, + gridDim.x, ...) arrive through a
// two-stage prefetch: the work entry (user, block) of the item after next and
// the per-user metadata of the next item are loaded one item ahead, so no
// role waits on a dependent pair of global loads at an item boundary.
struct ItemStream {
  int idx;
  int2 ub;                          // work entry of item idx + step
  int u, b;                         // item idx: work entry ...
  int32_t T, n;                     // ... and metadata (loads in flight)
  int64_t hoff, qoff;

  __device__ __forceinline__ static int2 entry(const AttnTcParams& p, int i, int n_items) {
    return i < n_items ? reinterpret_cast<const int2*>(p.work)[i] : make_int2(-1, 0);
  }
  __device__ __forceinline__ void fetch(const AttnTcParams& p, int2 e) {
    u = e.x;
    b = e.y;
    if (u >= 0) {
      T = p.T[u]; n = p.n[u]; hoff = p.hoff[u]; qoff = p.qoff[u];
    } else {
      T = n = 0; hoff = qoff = 0;
    }
  }
  __device__ __forceinline__ void start(const AttnTcParams& p, int first, int n_items, int step) {
    idx = first;
    fetch(p, entry(p, first, n_items));
    ub = entry(p, first + step, n_items);
  }
  // The current item, fully derived; then the prefetch moves one item on.
  // Block b covers (query row, head) pairs 128 b .. 128 b + 127 (heads
  // interleaved).
  __device__ __forceinline__ Item next(const AttnTcParams& p, int n_items, int step, int keys) {
    Item it;
    it.u = u; it.b = b; it.T = T; it.n = n; it.hoff = hoff; it.qoff = qoff;
    it.q = n + p.n_q;
    if (u < 0) {
      it.nk = 0;
    } else {
      const int64_t jl = min((int64_t)b * 128 + 127, (int64_t)it.q * p.heads - 1) / p.heads;
      const int64_t kmax = jl < n ? (int64_t)T - n + jl + 1 : T;
      it.nk = (int)((kmax + keys - 1) / keys);
    }
    fetch(p, ub);
    idx += step;
    ub = entry(p, idx + step, n_items);
    return it;
  }
};

// KP fp32 columns of this lane's TMEM row.
template <int KP>
__device__ __forceinline__ void tmem_ld_kp(uint32_t taddr, float (&v)[KP]) {
  if constexpr (KP == 64) tmem_ld64(taddr, v);
  else tmem_ld32(taddr, v);
}

// KP / 2 packed bf16 pairs into this lane's TMEM row.
template <int KP>
__device__ __forceinline__ void tmem_st_packed(uint32_t taddr, const uint32_t (&w)[KP / 2]) {
  if constexpr (KP == 64) {
    float f[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(w[i]);
    tmem_st32(taddr, f);          // waits for the store
  } else {
    tmem_st16u(taddr, w);
    tmem_wait_st();
  }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
               const AttnTcParams p) {
  using Cfg = AttnCfg<R>;
  constexpr int KEYS = Cfg::KEYS, KP = Cfg::KP, RSUB = Cfg::RSUB, KS = Cfg::KV_STAGES,
                OBUF = Cfg::OBUF, QBUF = Cfg::QBUF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + QBUF * Cfg::Q_BYTES;
  uint64_t* bars = (uint64_t*)(sKV + KS * Cfg::KV_BYTES);
  uint64_t* q_full = bars + 0;             // [2]
  uint64_t* q_empty = bars + 2;            // [2]
  uint64_t* kv_full = bars + 4;            // [KS]
  uint64_t* kv_empty = kv_full + KS;       // [KS]
  uint64_t* s_full = kv_empty + KS;        // [2]
  uint64_t* p_full = s_full + 2;           // [2] both halves of P(kt) written
  uint64_t* p_empty = p_full + 2;          // [2] P(kt) V done (O holds it)
  uint64_t* o_full = p_empty + 2;          // [OBUF] last PV done + row sums added
  uint64_t* o_free = o_full + 2;           // [OBUF] epilogue has read O
  uint64_t* pair_bar = o_free + 2;         // [4] the two softmax warps of a quadrant
  uint64_t* drain = pair_bar + 4;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* lbuf = (float*)((uint8_t*)bars + Cfg::BAR_BYTES);   // [2][128] row sums
  float* mx = lbuf + 2 * 128;                                  // [2][kSplit][128]
  uint8_t* sStage = (uint8_t*)(mx + 2 * kSplit * 128);         // [kEpiWarps][kStageBytes]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int step = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    for (int s = 0; s < KS; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], kSoftWarps);
      mbar_init(&p_empty[s], 1);
      mbar_init(&o_full[s], 1 + kSoftWarps);   // the MMA commit + every softmax warp
      mbar_init(&o_free[s], kEpiWarps);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&pair_bar[q], kSplit);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmC);
  }
  for (int i = threadIdx.x; i < 2 * 128; i += blockDim.x) lbuf[i] = 0.f;
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier kernels wrote
  pdl_wait();
  const int n_items = *p.work_count;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t itm = 0, g = 0, qi = 0;        // items, key tiles, query tiles issued
      bool ok = true;
      ItemStream items;
      items.start(p, blockIdx.x, n_items, step);
      for (int idx = blockIdx.x; idx < n_items && ok; idx += step) {
        const Item it = items.next(p, n_items, step, KEYS);
        if (it.nk == 0) continue;
        const int qb = itm % QBUF;
        if (!mbar_wait(&q_empty[qb], ((itm / QBUF) & 1) ^ 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&q_full[qb], Cfg::Q_BYTES);
        uint8_t* qdst = sQ + qb * Cfg::Q_BYTES;
        // 128 interleaved (row, head) pairs of r columns
        const int32_t qrow = (int32_t)(it.qoff * p.heads + (int64_t)it.b * 128);
#pragma unroll
        for (int s = 0; s < RSUB; ++s)
          tma_load_2d(&tmQ, &q_full[qb], qdst + s * 16384, s * 64, qrow);
        ++qi;
        for (int kt = 0; kt < it.nk; ++kt, ++g) {
          const int st = g % KS;
          if (!mbar_wait(&kv_empty[st], ((g / KS) & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], Cfg::KV_BYTES);
          const int32_t krow = (int32_t)(it.hoff + (int64_t)kt * KEYS);
          uint8_t* dst = sKV + st * Cfg::KV_BYTES;
#pragma unroll
          for (int s = 0; s < RSUB; ++s)
            tma_load_2d(&tmC, &kv_full[st], dst + s * Cfg::KV_SUB_BYTES, s * 64, krow);
        }
        ++itm;
      }
      // after an abort the MMA thread may have left key / query tiles unread
      if (*abort_flag) {
        drain_ring(kv_full, KS, g, p.status);
        drain_ring(q_full, QBUF, qi, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, KEYS, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, R, false, true);
      uint32_t itm = 0, g = 0;
      bool ok = true;
      // S(gg) into S buffer gg & 1.  That buffer last held P(gg - 2), whose
      // P V product was issued before this call, so the in-order tensor pipe
      // reads it first.
      auto issue_s = [&](uint32_t gg, uint32_t q_addr) -> bool {
        const int st = gg % KS;
        if (!mbar_wait(&kv_full[st], (gg / KS) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t kv_addr = smem_u32(sKV + st * Cfg::KV_BYTES);
        const uint32_t d = tmem + Cfg::S_COL + (gg & 1) * KEYS;
#pragma unroll
        for (int k = 0; k < R / 16; ++k) {
          const uint64_t ad = sdesc_sw128(q_addr + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
          const uint64_t bd =
              sdesc_sw128(kv_addr + (k >> 2) * Cfg::KV_SUB_BYTES + (k & 3) * 32, 16, 1024);
          umma_bf16(d, ad, bd, IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[gg & 1]);
        return true;
      };
      // PV of tile gg (item number `item`, O buffer ob); `first` zeroes O.
      // A = P(gg) from TMEM, B = the C tile read MN-major.
      auto issue_pv = [&](uint32_t gg, bool first, int ob, uint32_t item) -> bool {
        if (!mbar_wait(&p_full[gg & 1], (gg >> 1) & 1, abort_flag, p.status)) return false;
        // the O buffer of this item is free once the epilogue has read the
        // item that used it OBUF items ago
        if (first && !mbar_wait(&o_free[ob], ((item / OBUF) & 1) ^ 1, abort_flag, p.status))
          return false;
        tc_fence_after();
        const int st = gg % KS;
        const uint32_t kv_addr = smem_u32(sKV + st * Cfg::KV_BYTES);   // the same tile as V
        const uint32_t p_tmem = tmem + Cfg::S_COL + (gg & 1) * KEYS;
#pragma unroll
        for (int k = 0; k < KEYS / 16; ++k) {
          // 64-wide latent blocks are the sub-tiles (LBO apart), 16 keys per
          // MMA step = 2048 bytes
          const uint64_t bd = sdesc_sw128(kv_addr + k * 2048, Cfg::KV_SUB_BYTES, 1024);
          umma_bf16_ts(tmem + ob * R, p_tmem + p_col<KP>(k), bd, IDESC_O,
                       (!first || k > 0) ? 1u : 0u);
        }
        // the C tile is free, and (through p_empty) the softmax warps learn
        // that PV(gg) is in O
        umma_commit(&kv_empty[st]);
        umma_commit(&p_empty[gg & 1]);
        return true;
      };
      // The PV of a tile is issued after the S of the next tile, also across
      // item boundaries, so the softmax of tile g overlaps S(g + 1) even for
      // one-tile items.  `pend` is the tile whose PV is still to be issued.
      struct Pending { uint32_t g, item; int ob; bool first, last, valid; };
      Pending pend = {0, 0, 0, false, false, false};
      auto flush = [&]() -> bool {
        if (!pend.valid) return true;
        if (!issue_pv(pend.g, pend.first, pend.ob, pend.item)) return false;
        if (pend.last) umma_commit(&o_full[pend.ob]);   // every PV of that item is in O
        pend.valid = false;
        return true;
      };
      ItemStream items;
      items.start(p, blockIdx.x, n_items, step);
      for (int idx = blockIdx.x; idx < n_items && ok; idx += step) {
        const Item it = items.next(p, n_items, step, KEYS);
        if (it.nk == 0) continue;
        const int ob = itm % OBUF, qb = itm % QBUF;
        // with one query buffer the next block only arrives after the last S
        // of this one: finish the pending PV before waiting for it
        if (QBUF == 1 && !flush()) break;
        if (!mbar_wait(&q_full[qb], (itm / QBUF) & 1, abort_flag, p.status)) break;
        const uint32_t q_addr = smem_u32(sQ + qb * Cfg::Q_BYTES);
        for (int kt = 0; kt < it.nk; ++kt, ++g) {
          if (!issue_s(g, q_addr)) { ok = false; break; }
          if (kt == it.nk - 1) umma_commit(&q_empty[qb]);
          if (!flush()) { ok = false; break; }
          pend = {g, itm, ob, kt == 0, kt == it.nk - 1, true};
        }
        ++itm;
      }
      if (ok) flush();
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, &dummy, p.status);
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int part = (warp - 2) / 4;               // which half of the tile's keys
    const int row = quad * 32 + lane;              // pair within the block = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t g = 0, itm = 0, pphase = 0;
    bool ok = true;
    ItemStream items;
    items.start(p, blockIdx.x, n_items, step);
    for (int idx = blockIdx.x; idx < n_items && ok; idx += step) {
      const Item it = items.next(p, n_items, step, KEYS);
      if (it.nk == 0) continue;
      const int ob = itm % OBUF;
      const uint32_t o_col = ob * R + part * (R / 2);   // this warp's half of O
      // this lane's query row jl within the user (absorbed: of its pair)
      const int64_t pair = (int64_t)it.b * 128 + row;
      const bool valid = pair < (int64_t)it.q * p.heads;
      const int64_t jl = pair / p.heads;
      const int64_t vis = !valid ? 0 : (jl < it.n ? (int64_t)it.T - it.n + jl + 1 : it.T);
      float m_run = -INFINITY, l_run = 0.f;   // running max (log2 domain) and partial sum
      for (int kt = 0; kt < it.nk; ++kt, ++g) {
        // ---- masked row max over this warp's keys.  Scores are already in
        // log2 units (log2 e folded into q~).
        bool w = mbar_wait(&s_full[g & 1], (g >> 1) & 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_addr = lane_base + Cfg::S_COL + (g & 1) * KEYS + part * KP;
        // keys [0, lim) of this warp's KP are visible to the row; masking is
        // applied only when some row of the warp stops inside them.  Rows past
        // the user's last query row (the padding of its last block) are never
        // stored, so they take every key and do not force the masked path.
        const int64_t lim64 = vis - (int64_t)kt * KEYS - part * KP;
        const int lim = !valid ? KP : (lim64 <= 0 ? 0 : (lim64 >= KP ? KP : (int)lim64));
        const bool masked = __any_sync(0xffffffffu, lim < KP);
        float v[KP];
        tmem_ld_kp<KP>(s_addr, v);
        if (masked) {
#pragma unroll
          for (int i = 0; i < KP; ++i) v[i] = (i < lim) ? v[i] : -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
#pragma unroll
        for (int i = 0; i < KP; i += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], v[i + k], v[i + 8 + k]);
        }
        float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                         fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        // the two halves of the row meet: both warps end with the same max
        float* mxs = mx + (g & 1) * kSplit * 128;
        mxs[part * 128 + row] = mt;
        if (!group_sync(&pair_bar[quad], pphase, abort_flag, p.status)) { ok = false; break; }
        mt = fmaxf(mt, mxs[(part ^ 1) * 128 + row]);
        // ---- lazy rescale of O and l (only when the max grows by > 8 in log2);
        // both warps of the quadrant take the same decisions
        float scale = 1.f;
        bool resc = false;
        if (kt == 0) {
          m_run = mt;
        } else if (mt > m_run + 8.f) {
          scale = ex2_approx(m_run - mt);
          m_run = mt;
          resc = true;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // PV(g-1) must have landed in O before O is touched.  Its completion
          // is the next phase of p_empty[(g-1)&1]: that barrier cannot run a
          // phase further ahead because PV(g+1) needs P(g+1), not written yet.
          bool w2 = mbar_wait(&p_empty[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, p.status);
          if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < R / 2; c += 32) {
            float o[32];
            tmem_ld32(lane_base + o_col + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= scale;
            tmem_st32(lane_base + o_col + c, o);
          }
          l_run *= scale;
        }
        // ---- probabilities 2^(s - m) -> bf16, written over S in TMEM.  One
        // pair in eight takes the FMA-pipe exponential, the rest the special-
        // function unit; both give exactly 0 for a masked score (-inf).  A
        // row that sees no key at all keeps m = -inf and subtracts 0 instead.
        const float m_use = m_run > -INFINITY ? m_run : 0.f;
        const float2 nm2 = make_float2(-m_use, -m_use);
#pragma unroll
        for (int j = 0; j < KP / 2; ++j) {
          float2 x = add_f2(make_float2(v[2 * j], v[2 * j + 1]), nm2);
          // one pair in eight on the FMA pipe
          if ((j & 7) == 7) {
            x = exp2_fma2(x);
          } else {
            x.x = ex2_approx(x.x);
            x.y = ex2_approx(x.y);
          }
          v[2 * j] = x.x;
          v[2 * j + 1] = x.y;
        }
        float2 l4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) l4[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < KP / 2; ++j)
          l4[j & 3] = add_f2(l4[j & 3], make_float2(v[2 * j], v[2 * j + 1]));
        l_run += ((l4[0].x + l4[0].y) + (l4[1].x + l4[1].y)) +
                 ((l4[2].x + l4[2].y) + (l4[3].x + l4[3].y));
        uint32_t pk[KP / 2];
#pragma unroll
        for (int j = 0; j < KP / 2; ++j) pk[j] = pack_bf16(v[2 * j], v[2 * j + 1]);
        tmem_st_packed<KP>(s_addr, pk);
        // P(g) half written: the MMA may read it once both halves are in
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g & 1]);
      }
      if (!ok) break;
      // ---- add this half's row sum for the epilogue warps (the sum slot of
      // this O buffer is free, and zero, once the epilogue has finished the
      // item OBUF ago)
      bool w4 = mbar_wait(&o_free[ob], ((itm / OBUF) & 1) ^ 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w4)) break;
      atomicAdd(&lbuf[ob * 128 + row], l_run);
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_full[ob]);
      ++itm;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t stg = smem_u32(sStage + (warp - kEpiWarp0) * kStageBytes);
    uint32_t itm = 0;
    ItemStream items;
    items.start(p, blockIdx.x, n_items, step);
    for (int idx = blockIdx.x; idx < n_items; idx += step) {
      const Item it = items.next(p, n_items, step, KEYS);
      const int64_t pair = (int64_t)it.b * 128 + row;
      __nv_bfloat16* orow =
          pair < (int64_t)it.q * p.heads ? p.Ot + (it.qoff * p.heads + pair) * R : nullptr;
      if (it.nk == 0) {                 // no key: the attention output is zero
        const uint4 z[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                            make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        for (int c = 0; c < R; c += 32) stage_store(stg, z, orow ? orow + c : nullptr);
        continue;
      }
      const int ob = itm % OBUF;
      bool w = mbar_wait(&o_full[ob], (itm / OBUF) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const float l = lbuf[ob * 128 + row];
      lbuf[ob * 128 + row] = 0.f;        // ready for the item that reuses this buffer
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < R; c += 64) {
        float v[64];
        tmem_ld64(lane_base + ob * R + c, v);
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] *= inv;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 x[4];
          pack_bf16x32(&v[32 * h], x);
          stage_store(stg, x, orow ? orow + c + 32 * h : nullptr);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[ob]);
      ++itm;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

template <int R>
cudaError_t launch_r(const CUtensorMap& q, const CUtensorMap& c, const AttnTcParams& p, int grid,
                     cudaStream_t s) {
  using Cfg = AttnCfg<R>;
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg::SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  return launch_dependent(attn_tc_kernel<R>, dim3(grid), dim3(kThreads), Cfg::SMEM, s, 1, q,
                          c, p);
}

}  // namespace

int attn_tc_keys(int) { return 128; }

bool attn_tc_supported(int r) { return r == 64 || r == 128 || r == 256; }

cudaError_t launch_attn_tc(int r, const CUtensorMap& q, const CUtensorMap& c,
                           const AttnTcParams& p, int num_sms, cudaStream_t s) {
  const int grid = std::max(1, std::min(num_sms, p.max_items));
  switch (r) {
    case 64: return launch_r<64>(q, c, p, grid, s);
    case 128: return launch_r<128>(q, c, p, grid, s);
    case 256: return launch_r<256>(q, c, p, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace llatte
