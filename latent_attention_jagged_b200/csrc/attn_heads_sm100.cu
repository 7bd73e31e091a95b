// Fused attention for sm_100a, MLA in its per-head form (LLaTTE notes,
// huaxiaozhuan.com, appendix A.3 first display: K, V = split(c_kv W_up^KV),
// scores over d_h = 64; target-aware causal / candidate masking of appendix
// A.2): per query row and head, s_t = q . k_t over the visible keys,
// softmax, o = sum_t a_t v_t.
//
// At d_h = 64 the work per 128 x 128 tile is four S products of N = 128 and
// eight P V products of N = 64, which the tensor pipe runs one after the
// other at a fixed cost each, so the kernel is built to keep that pipe fed:
// two CTAs per SM, each with one 128-row query tile at a time, so that one
// CTA's products run while the other CTA's softmax works (the SM interleaves
// the two CTAs' product streams).  Per CTA:
//   TMEM   O | S | P        (64 + 128 + 64 = 256 columns, half of the SM's)
// P is kept apart from S, so S(kt + 1) is computed while the softmax still
// turns the scores of tile kt into probabilities: the softmax signals "S
// read" once its TMEM loads of the scores are done and the row max is known,
// and the MMA issuer starts S(kt + 1) then; O += P(kt) V follows once P(kt)
// is written.
//
// Work item: one user, one head and a block of 128 query rows (the attention
// work list of the layer, ordered by user).
// Roles (320 threads):
//   warp 0       TMA: the item's query tile (double-buffered, so the next
//                item's arrives during this one), then its key and value tiles
//                into a 2-stage ring
//   warp 1       TMEM owner; lane 0 issues, per key tile, S(kt) once the
//                softmax has read S(kt - 1), then O += P(kt - 1) V once P(kt - 1)
//                is written
//   warps 2..9   softmax, two warps per TMEM lane quadrant, each taking 64 of
//                the tile's 128 keys for the quadrant's 32 rows (one row per
//                thread), 32 keys at a time; past an item's first tile in one
//                pass (probabilities against the running max, the tile max on
//                the side), the two warps' maxima meeting in shared memory
//                behind a bounded pair barrier; a second pass only on an
//                item's first tile or when a row's max grows by more than 2^8
//                (then O and l are rescaled).  Masking: a history row at
//                position p sees keys t <= p, a query token every key t < T.
//                P goes to TMEM as bf16 16 columns at a time once the previous
//                P V product has read it.  The same warps divide O by the row
//                sums (each warp 32 of its 64 columns) and store it straight
//                from registers, deferred into the next item's first tile so
//                that the softmax never waits for the last product of an item.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_attn.h"
#include "tc_common.cuh"
#include "tc_epilogue.cuh"

namespace llatte {

using namespace tc;

namespace {

constexpr int kSplit = 2;                          // softmax warps per TMEM lane quadrant
constexpr int kSoftWarps = 4 * kSplit;
constexpr int kThreads = 32 * (2 + kSoftWarps);
constexpr int KEYS = 128;                          // keys per tile
constexpr int KP = KEYS / kSplit;                  // keys per softmax warp
constexpr int DH = 64;                             // head width
constexpr int QBUF = 2;                            // query tiles in flight
constexpr int KS = 2;                              // key / value tiles in the ring
constexpr uint32_t Q_BYTES = 128 * DH * 2;         // 16 KB
constexpr uint32_t KV_BYTES = 2 * KEYS * DH * 2;   // K tile + V tile, 32 KB
constexpr uint32_t V_OFF = KEYS * DH * 2;
constexpr uint32_t O_COL = 0;
constexpr uint32_t S_COL = DH;
constexpr uint32_t P_COL = S_COL + KEYS;           // bf16 pairs: keys 2j, 2j + 1 in column j
constexpr uint32_t TMEM_COLS = 256;
static_assert(P_COL + KEYS / 2 <= TMEM_COLS, "TMEM budget");
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t MX_BYTES = 2 * kSplit * 128 * 4;   // partial row maxima, by tile parity
constexpr uint32_t LX_BYTES = kSplit * 128 * 4;       // partial row sums at an item's end
constexpr size_t SMEM = 1024 + QBUF * Q_BYTES + (size_t)KS * KV_BYTES + BAR_BYTES + MX_BYTES +
                        LX_BYTES;
// two CTAs per SM
static_assert(2 * (SMEM + 1024) <= 233472, "shared memory budget");

struct Item {
  int u, b;
  int32_t T, n, q;
  int nk;            // key tiles (0: no key at all)
  int64_t hoff, qoff;
};

// Work entries (user, 128-row block * heads + head) arrive through a
// two-stage prefetch, so no role waits on a dependent pair of global loads
// at an item boundary.
struct ItemStream {
  int idx;
  int2 ub;
  int u, b;
  int32_t T, n;
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
  __device__ __forceinline__ Item next(const AttnTcParams& p, int n_items, int step) {
    Item it;
    it.u = u; it.b = b; it.T = T; it.n = n; it.hoff = hoff; it.qoff = qoff;
    it.q = n + p.n_q;
    it.nk = 0;
    if (u >= 0) {
      // keys visible to the block's last row
      const int64_t jl = min((int64_t)(b / p.heads) * 128 + 127, (int64_t)it.q - 1);
      const int64_t kmax = jl < n ? (int64_t)T - n + jl + 1 : T;
      it.nk = (int)((kmax + KEYS - 1) / KEYS);
    }
    fetch(p, ub);
    idx += step;
    ub = entry(p, idx + step, n_items);
    return it;
  }
};

// Largest growth of the running max (log2 domain) that the one-pass softmax
// absorbs without rescaling: the probabilities of a tile stay below 2^kGrow.
constexpr float kGrow = 8.f;

// Keys at or past lim of these 32 take -inf.
__device__ __forceinline__ void mask_keys(float (&v)[32], int lim) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = i < lim ? v[i] : -INFINITY;
}
// Four running maxima over 32 scores (three-input max).
__device__ __forceinline__ void max_keys(float (&m4)[4], const float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) m4[k] = fmax3(m4[k], v[i + k], v[i + 4 + k]);
  }
}
// 2^(s - m) for 32 scores: bf16 pairs (keys 2j, 2j + 1 in word j) and the
// fp32 sums of four interleaved partial rows (two packed pairs).
__device__ __forceinline__ void exp_keys(const float (&v)[32], float m, float2 (&l2)[2],
                                         uint32_t (&pk)[16]) {
  const float2 nm2 = make_float2(-m, -m);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float2 x = add_f2(make_float2(v[2 * j], v[2 * j + 1]), nm2);
    x.x = ex2_approx(x.x);
    x.y = ex2_approx(x.y);
    l2[j & 1] = add_f2(l2[j & 1], x);
    pk[j] = pack_bf16(x.x, x.y);
  }
}

// 16 packed probability words into TMEM (one lane's row), waiting for the store.
__device__ __forceinline__ void store_p(uint32_t taddr, const uint32_t (&pk)[16]) {
  tmem_st16u(taddr, pk);
  tmem_wait_st();
}

// Wait for a phase without giving up on the CTA's abort flag (drains only):
// still bounded by the default wait limit.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
  int never = 0;
  mbar_wait(bar, parity, &never, status);
}

__global__ void __launch_bounds__(kThreads, 2)
attn_heads_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                  const AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                             // [QBUF][Q_BYTES]
  uint8_t* sKV = sQ + QBUF * Q_BYTES;             // [KS][KV_BYTES]
  uint64_t* bars = (uint64_t*)(sKV + KS * KV_BYTES);
  uint64_t* q_full = bars;                        // [QBUF]
  uint64_t* q_empty = q_full + QBUF;              // [QBUF]
  uint64_t* kv_full = q_empty + QBUF;             // [KS]
  uint64_t* kv_empty = kv_full + KS;              // [KS]
  uint64_t* s_full = kv_empty + KS;               // S(kt) in TMEM
  uint64_t* s_free = s_full + 1;                  // the softmax has read S(kt)
  uint64_t* p_full = s_free + 1;                  // P(kt) written
  uint64_t* pv_done = p_full + 1;                 // O += P(kt) V done (P free)
  uint64_t* o_free = pv_done + 1;                 // the previous item's O has been read
  uint64_t* drain = o_free + 1;
  uint64_t* never = drain + 1;                    // nothing arrives (injected timeout)
  uint64_t* pair_bar = never + 1;                 // [4] the two softmax warps of a quadrant
  uint32_t* tmem_slot = (uint32_t*)(pair_bar + 4);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  static_assert((2 * QBUF + 2 * KS + 11) * 8 + 8 <= BAR_BYTES, "barrier area");
  float* mx = (float*)((uint8_t*)bars + BAR_BYTES);    // [2][kSplit][128]
  float* lx = mx + 2 * kSplit * 128;                   // [kSplit][128]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int step = gridDim.x;
  const uint64_t lim = kWaitTimeoutNs;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QBUF; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1); }
    for (int s = 0; s < KS; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftWarps);
    mbar_init(p_full, kSoftWarps);
    mbar_init(pv_done, 1);
    mbar_init(o_free, kSoftWarps);
    mbar_init(drain, 1);
    mbar_init(never, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&pair_bar[i], kSplit);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
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
      uint32_t qi = 0, g = 0;          // query tiles, key tiles loaded
      bool ok = true;
      ItemStream items;
      items.start(p, blockIdx.x, n_items, step);
      for (int idx = blockIdx.x; idx < n_items && ok; idx += step) {
        const Item it = items.next(p, n_items, step);
        if (it.nk == 0) continue;
        const int head = it.b % p.heads;
        const int qb = (int)(qi % QBUF);
        if (!mbar_wait(&q_empty[qb], ((qi / QBUF) & 1) ^ 1, abort_flag, p.status, lim)) break;
        mbar_arrive_expect_tx(&q_full[qb], Q_BYTES);
        tma_load_2d(&tmQ, &q_full[qb], sQ + qb * Q_BYTES, head * DH,
                    (int32_t)(it.qoff + (int64_t)(it.b / p.heads) * 128));
        ++qi;
        for (int kt = 0; kt < it.nk; ++kt, ++g) {
          const int st = g % KS;
          if (!mbar_wait(&kv_empty[st], ((g / KS) & 1) ^ 1, abort_flag, p.status, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[st], KV_BYTES);
          const int32_t krow = (int32_t)(it.hoff + (int64_t)kt * KEYS);
          uint8_t* dst = sKV + st * KV_BYTES;
          // K then V of this head: columns 64 j and h * 64 + 64 j
          tma_load_2d(&tmKV, &kv_full[st], dst, head * DH, krow);
          tma_load_2d(&tmKV, &kv_full[st], dst + V_OFF, (p.heads + head) * DH, krow);
        }
      }
      // no load may still be landing in shared memory when the CTA exits:
      // wait for the last key tiles and query tiles issued (they complete on
      // their own; the waits are bounded all the same)
      for (uint32_t k = 0; k < (uint32_t)KS && k < g; ++k) {
        const uint32_t gg = g - 1 - k;
        drain_wait(&kv_full[gg % KS], (gg / KS) & 1, p.status);
      }
      for (uint32_t k = 0; k < (uint32_t)QBUF && k < qi; ++k) {
        const uint32_t qq = qi - 1 - k;
        drain_wait(&q_full[qq % QBUF], (qq / QBUF) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, KEYS, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16(128, DH, false, true);
      uint32_t qi = 0, g = 0;          // query tiles, key tiles consumed (= S products)
      uint32_t pc = 0, oi = 0;         // P V products issued, items with keys started
      bool inject = p.inject_timeout != 0;
      bool ok = true;
      // the P V product still to be issued
      struct Pending { int st; bool first, valid; };
      Pending pend = {0, false, false};
      auto flush = [&]() -> bool {
        if (!pend.valid) return true;
        if (inject) {
          // failure-detection test: with an S product and key tiles in
          // flight, wait on a barrier that nothing arrives on, with a short
          // limit; the wait runs out, records the timeout and winds the CTA
          // down
          inject = false;
          if (!mbar_wait(never, 0, abort_flag, p.status, 20000)) return false;
        }
        if (!mbar_wait(p_full, pc & 1, abort_flag, p.status, lim)) return false;
        // the first product of an item overwrites O: the softmax must have
        // read the previous item's O
        if (pend.first && !mbar_wait(o_free, (oi & 1) ^ 1, abort_flag, p.status, lim)) return false;
        if (pend.first) ++oi;
        ++pc;
        tc_fence_after();
        const uint64_t bd0 =
            sdesc_sw128(smem_u32(sKV + pend.st * KV_BYTES) + V_OFF, KEYS * 128, 1024);
#pragma unroll
        for (int k = 0; k < KEYS / 16; ++k)
          // 16 keys per MMA step = 2048 bytes of V (MN-major), 8 packed P columns
          umma_bf16_ts(tmem + O_COL, tmem + P_COL + 8 * k, bd0 + (uint64_t)(128 * k), IDESC_O,
                       (!pend.first || k > 0) ? 1u : 0u);
        umma_commit(pv_done);
        umma_commit(&kv_empty[pend.st]);
        pend.valid = false;
        return true;
      };
      ItemStream items;
      items.start(p, blockIdx.x, n_items, step);
      for (int idx = blockIdx.x; idx < n_items && ok; idx += step) {
        const Item it = items.next(p, n_items, step);
        if (it.nk == 0) continue;
        const int qb = (int)(qi % QBUF);
        for (int kt = 0; kt < it.nk; ++kt, ++g) {
          const int st = g % KS;
          // S(g) once the softmax has read S(g - 1), the key tile is in and
          // (first tile of the item) the query tile
          if (g > 0 && !mbar_wait(s_free, (g - 1) & 1, abort_flag, p.status, lim)) { ok = false; break; }
          if (!mbar_wait(&kv_full[st], (g / KS) & 1, abort_flag, p.status, lim)) { ok = false; break; }
          if (kt == 0) {
            if (!mbar_wait(&q_full[qb], (qi / QBUF) & 1, abort_flag, p.status, lim)) { ok = false; break; }
            ++qi;
          }
          tc_fence_after();
          const uint64_t ad0 = sdesc_sw128(smem_u32(sQ + qb * Q_BYTES), 16, 1024);
          const uint64_t bd0 = sdesc_sw128(smem_u32(sKV + st * KV_BYTES), 16, 1024);
#pragma unroll
          for (int k = 0; k < DH / 16; ++k)   // 16 head dims = 32 bytes per step
            umma_bf16(tmem + S_COL, ad0 + (uint64_t)(2 * k), bd0 + (uint64_t)(2 * k), IDESC_S,
                      k > 0 ? 1u : 0u);
          umma_commit(s_full);
          if (kt == it.nk - 1) umma_commit(&q_empty[qb]);
          // then the P V product of the previous key tile
          if (!flush()) { ok = false; break; }
          pend = {st, kt == 0, true};
        }
      }
      if (ok) flush();
      // every MMA of this CTA must be complete before TMEM is released
      umma_commit(drain);
      drain_wait(drain, 0, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int sw = warp - 2;
    const int quad = warp & 3;                       // TMEM lane quadrant
    const int part = sw >> 2;                        // which KP keys of the tile, O columns
    const int row = quad * 32 + lane;                // row within the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t s_base = lane_base + S_COL + part * KP;
    const uint32_t p_base = lane_base + P_COL + part * (KP / 2);
    const uint32_t o_base = lane_base + O_COL + part * (DH / 2);
    uint32_t sc = 0, pphase = 0;
    bool ok = true;
    // The epilogue of an item is deferred into the next item's first tile:
    // its O is read once the P V product before that tile's P is done (the
    // wait that tile makes anyway) and that P is handed over (the first
    // product of the new item also waits for o_free), so the softmax never
    // stalls for the last product of an item.  The row (this warp's 32
    // columns of it) and 1 / l of that item:
    __nv_bfloat16* prev_orow = nullptr;
    float prev_inv = 0.f;
    bool prev_pending = false;
    // O / l of the pending item -> 32 bf16 columns of the row (O holds its
    // last product); 64 bytes per lane, straight from registers
    auto finish_prev = [&]() {
      float o[32];
      tmem_ld32(o_base, o);
      // O may take the next item's first product
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= prev_inv;
      uint4 x[4];
      pack_bf16x32(o, x);
      if (prev_orow) {
        uint4* dst = reinterpret_cast<uint4*>(prev_orow);
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[c] = x[c];
      }
      prev_pending = false;
    };
    ItemStream items;
    items.start(p, blockIdx.x, n_items, step);
    for (int idx = blockIdx.x; idx < n_items && ok; idx += step) {
      const Item it = items.next(p, n_items, step);
      // this lane's query row jl within the user, and where this warp's 32
      // output columns go (null: padding past the user's last row)
      const int64_t jl = (int64_t)(it.b / p.heads) * 128 + row;
      const bool valid = it.u >= 0 && jl < (int64_t)it.q;
      __nv_bfloat16* orow = valid ? p.Ot + (it.qoff + jl) * (int64_t)(p.heads * DH) +
                                        (it.b % p.heads) * DH + part * (DH / 2)
                                  : nullptr;
      if (it.nk == 0) {                 // no key at all: the attention output is zero
        if (orow) {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const int64_t vis = !valid ? 0 : (jl < it.n ? (int64_t)it.T - it.n + jl + 1 : it.T);
      // running max (log2 domain; the same in both warps of the quadrant)
      // and this warp's part of the row sum
      float m_run = -INFINITY, l_run = 0.f;
      for (int kt = 0; kt < it.nk; ++kt) {
        bool w = mbar_wait(s_full, sc & 1, abort_flag, p.status, lim);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        // keys [0, lim_k) of this warp's KP are visible to the row; masking
        // only when some row of the warp stops inside them.  Padding rows take
        // every key (they are never stored).
        const int64_t lim64 = vis - (int64_t)kt * KEYS - part * KP;
        const int lim_k = !valid ? KP : (lim64 <= 0 ? 0 : (lim64 >= KP ? KP : (int)lim64));
        const bool masked = __any_sync(0xffffffffu, lim_k < KP);
        // One pass over the scores, 32 keys at a time: the row max on the
        // side and, past the item's first tile, the probabilities 2^(s - m)
        // against the running max m (they may exceed 1 until m catches up, by
        // at most 2^kGrow).  The two warps of the quadrant then agree on the
        // row max; on the item's first tile (no m yet), or when that max
        // exceeds m by more than kGrow in some row, both take a second pass
        // with the new max instead.  Every exponential goes to the special-
        // function unit: the softmax is bound by issue slots, and the FMA-pipe
        // form costs seven times the instructions.  A masked score (-inf)
        // gives exactly 0; a row that sees no key keeps m = -inf and
        // subtracts 0 instead.
        const bool have_m = kt > 0;
        const float m_use = m_run > -INFINITY ? m_run : 0.f;
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // P and O are free once the previous P V product is done
        bool pv_waited = sc == 0;
        auto wait_pv = [&]() -> bool {
          if (pv_waited) return true;
          pv_waited = true;
          const bool w2 = mbar_wait(pv_done, (sc - 1) & 1, abort_flag, p.status, lim);
          if (!__all_sync(0xffffffffu, w2)) return false;
          tc_fence_after();
          return true;
        };
        {
          float v[32];
          tmem_ld32(s_base, v);
          if (masked) mask_keys(v, lim_k);
          max_keys(m4, v);
          if (have_m) {
            uint32_t pk[16];
            exp_keys(v, m_use, l2, pk);
            if (!wait_pv()) { ok = false; break; }
            store_p(p_base, pk);
          }
        }
        float v[32];
        tmem_ld32(s_base + 32, v);
        if (masked) mask_keys(v, lim_k - 32);
        max_keys(m4, v);
        float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        // the row max over both halves of the tile
        float* mxs = mx + (sc & 1) * kSplit * 128;
        mxs[part * 128 + row] = mt;
        if (!group_sync(&pair_bar[quad], pphase, abort_flag, p.status)) { ok = false; break; }
        mt = fmaxf(mt, mxs[(part ^ 1) * 128 + row]);
        const bool redo = !have_m || __any_sync(0xffffffffu, mt > m_use + kGrow);
        float scale = 1.f;
        bool resc = false;
        if (!redo) {
          // the scores are in registers: S may take the next tile
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
          uint32_t pk[16];
          exp_keys(v, m_use, l2, pk);
          if (!wait_pv()) { ok = false; break; }
          store_p(p_base + 16, pk);
        } else {
          // the new max: O and l rescaled (O once the previous P V product
          // is in it, below)
          if (mt > m_run) {
            if (have_m) {
              scale = ex2_approx(m_run - mt);
              resc = true;
            }
            m_run = mt;
          }
          const float m_new = m_run > -INFINITY ? m_run : 0.f;
          l2[0] = l2[1] = make_float2(0.f, 0.f);
          if (!wait_pv()) { ok = false; break; }
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float u[32];
            tmem_ld32(s_base + 32 * c, u);
            if (c == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(s_free);
            }
            if (masked) mask_keys(u, lim_k - 32 * c);
            uint32_t pk[16];
            exp_keys(u, m_new, l2, pk);
            store_p(p_base + 16 * c, pk);
          }
        }
        l_run = l_run * scale + ((l2[0].x + l2[0].y) + (l2[1].x + l2[1].y));
        if (!wait_pv()) { ok = false; break; }
        ++sc;
        if (__any_sync(0xffffffffu, resc)) {
          float o[32];
          tmem_ld32(o_base, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= scale;
          tmem_st32(o_base, o);
        }
        // P(kt) written: the MMA may read it once the eight warps are in
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // first tile of an item: the previous item's O is complete (the
        // product waited for above); this item's first product waits for o_free
        if (prev_pending) finish_prev();
      }
      if (!ok) break;
      // the row sum over both halves; this item's epilogue waits for the next
      // item's first tile (or the end)
      lx[part * 128 + row] = l_run;
      if (!group_sync(&pair_bar[quad], pphase, abort_flag, p.status)) { ok = false; break; }
      const float l_row = l_run + lx[(part ^ 1) * 128 + row];
      prev_orow = orow;
      prev_inv = l_row > 0.f ? 1.f / l_row : 0.f;
      prev_pending = true;
    }
    if (ok && prev_pending) {
      // the last item: its final P V product, then its rows
      bool w = mbar_wait(pv_done, (sc - 1) & 1, abort_flag, p.status, lim);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        finish_prev();
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attn_heads(const CUtensorMap& q, const CUtensorMap& kv, const AttnTcParams& p,
                              int num_sms, cudaStream_t s) {
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(attn_heads_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  // two CTAs per SM
  const int grid = std::max(1, std::min(2 * num_sms, p.max_items));
  return launch_dependent(attn_heads_kernel, dim3(grid), dim3(kThreads), SMEM, s, 1, q, kv, p);
}

}  // namespace llatte
