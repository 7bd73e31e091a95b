// Pyramid plan and jagged gather.
//
// Plan (LLaTTE notes, huaxiaozhuan.com, appendix A.2 "Transformer Layers and
// Pyramidal Schedule"): per user u and layer l, T_{0,u} = offsets[u+1] -
// offsets[u]; n_{l,u} = min(T_{l,u}, keep_l); T_{l+1,u} = n_{l,u}.  History
// (key) rows of layer l are packed per user in hist_off_l = exscan(T_l); its
// query rows (the last n_l history rows, then the n_q query tokens, i.e. the
// pages' tail slice of the fused sequence) in query_off_l = exscan(n_l + n_q).
// The layer after the last one is a virtual layer L whose keep is unbounded:
// its query rows are the final rows.  One CTA per layer; the offsets are
// validated first and a bad batch turns every count to zero (no later kernel
// then does any work) and sets the device status word.
//
// Gather (appendix A.2 step 2, X_input = Concat(X_seq, Q)): layer 0's
// history rows are a copy of `values`; its query rows are the last n_0
// history rows of each user followed by the user's query tokens.  Blocks per
// (user, slice), one warp per row, 16-byte vector loads/stores.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace llatte {

struct KeepArr { int32_t k[LLATTE_MAX_LAYERS + 1]; };

constexpr int kPlanThreads = 1024;

// Block-wide exclusive scan of two int64 values (one per thread).
__device__ void block_exscan2(int64_t a, int64_t b, int64_t* out_a, int64_t* out_b,
                              int64_t* tot_a, int64_t* tot_b) {
  __shared__ int64_t wa[32], wb[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t ta = __shfl_up_sync(0xffffffffu, ia, o);
    int64_t tb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += ta; ib += tb; }
  }
  if (lane == 31) { wa[warp] = ia; wb[warp] = ib; }
  __syncthreads();
  if (warp == 0) {
    int64_t xa = wa[lane], xb = wb[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t ta = __shfl_up_sync(0xffffffffu, xa, o);
      int64_t tb = __shfl_up_sync(0xffffffffu, xb, o);
      if (lane >= o) { xa += ta; xb += tb; }
    }
    wa[lane] = xa; wb[lane] = xb;
  }
  __syncthreads();
  int64_t pa = warp ? wa[warp - 1] : 0, pb = warp ? wb[warp - 1] : 0;
  *out_a = pa + ia - a;
  *out_b = pb + ib - b;
  *tot_a = wa[31];
  *tot_b = wb[31];
  __syncthreads();
}

// Block l handles layer l (block L the virtual final layer): every layer's
// counts have a closed form in the input length, T_{l,u} = min(T_{0,u},
// keep_0, ..., keep_{l-1}), so the layers need not wait for one another.
__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int64_t* __restrict__ offsets, int B, PlanDev p, KeepArr keep, int L, int n_q,
            int64_t max_len, int64_t max_total, int heads, int attn_keys, uint32_t heads_mask) {
  __shared__ int s_err;
  const int tid = threadIdx.x;
  const int l = blockIdx.x;
  if (tid == 0) s_err = 0;
  __syncthreads();
  int err = 0;
  for (int u = tid; u < B; u += kPlanThreads) {
    int64_t a = offsets[u], b = offsets[u + 1];
    if (a < 0 || b < a) err |= LLATTE_DEV_BAD_OFFSETS;
    else if (b - a > max_len) err |= LLATTE_DEV_TOO_LONG;
  }
  if (err) atomicOr(&s_err, err);
  __syncthreads();
  if (tid == 0 && s_err == 0 && offsets[B] - offsets[0] > max_total)
    s_err |= LLATTE_DEV_TOO_MANY_ROWS;
  __syncthreads();
  if (s_err) {
    // every block clears its own layer; block 0 reports
    if (tid == 0) {
      if (l == 0) atomicOr(p.status, s_err);
      p.totals[2 * l] = 0;
      p.totals[2 * l + 1] = 0;
      if (l < L) p.work_count[l] = 0;
    }
    for (int64_t i = tid; i < p.stride; i += kPlanThreads) {
      p.hist_off[l * p.stride + i] = 0;
      p.query_off[l * p.stride + i] = 0;
    }
    return;
  }
  int32_t cap = 0x7fffffff;                  // min of the keeps of the layers before l
  for (int k = 0; k < l; ++k) cap = min(cap, keep.k[k]);
  const int32_t kl = l < L ? keep.k[l] : 0x7fffffff;
  const int chunk = (B + kPlanThreads - 1) / kPlanThreads;
  const int u0 = min(B, tid * chunk), u1 = min(B, u0 + chunk);
  const int64_t bstride = p.stride - 1;
  {
    int32_t* Tl = p.T + l * bstride;
    int32_t* nl = p.n + l * bstride;
    int64_t sT = 0, sQ = 0;
    for (int u = u0; u < u1; ++u) {
      const int64_t len = offsets[u + 1] - offsets[u];
      const int32_t t = (int32_t)(len < cap ? len : cap);
      const int32_t nn = min(t, kl);
      Tl[u] = t;
      nl[u] = nn;
      sT += t;
      sQ += nn + n_q;
    }
    int64_t bT, bQ, totT, totQ;
    block_exscan2(sT, sQ, &bT, &bQ, &totT, &totQ);
    int64_t* ho = p.hist_off + l * p.stride;
    int64_t* qo = p.query_off + l * p.stride;
    for (int u = u0; u < u1; ++u) {
      ho[u] = bT;
      qo[u] = bQ;
      bT += Tl[u];
      bQ += nl[u] + n_q;
    }
    if (tid == 0) {
      ho[B] = totT;
      qo[B] = totQ;
      p.totals[2 * l] = totT;
      p.totals[2 * l + 1] = totQ;
    }
  }
  __syncthreads();
  if (attn_keys <= 0 || l == L) return;

  // Attention work list of layer l: one item per (user, block of 128 (query
  // row, head) pairs) -- or, for a layer in the per-head form (bit l of
  // heads_mask), per (user, 128-row block, head) with b = block * heads + head
  // -- ordered by the number of key tiles the block visits, largest first (a
  // counting sort over at most kBuckets cost classes), so that the persistent
  // attention CTAs take the longest items first.  A per-head layer orders its
  // items by user instead (users with the most key tiles first; within a
  // user head by head, the longest block first), so that the blocks of one
  // (user, head), which read the same key and value tiles, run at the same
  // time on neighbouring CTAs and share those tiles through L2 (ordered by
  // cost, all users' blocks of one cost class ran together and their key /
  // value tiles did not fit in L2).
  constexpr int kBuckets = 64;
  __shared__ int32_t hist[kBuckets], cursor[kBuckets];
  __shared__ int32_t total_items;
  // the users' first items, also in shared memory for batches of at most
  // kSmemUsers users: every item finds its user by a binary search over them,
  // which in global memory is a chain of dependent L2 round trips
  constexpr int kSmemUsers = 4096;
  __shared__ int32_t s_item_off[kSmemUsers + 1];
  const bool off_smem = B <= kSmemUsers;
  const int32_t* Tl = p.T + l * bstride;
  const int32_t* nl = p.n + l * bstride;
  int32_t* item_off = p.item_off + l * p.stride;
  const bool per_head = (heads_mask >> l) & 1u;
  auto items_of = [&](int u) -> int64_t {
    const int64_t q = (int64_t)nl[u] + n_q;
    return per_head ? ((q + 127) / 128) * heads : (q * heads + 127) / 128;
  };
  if (tid < kBuckets) hist[tid] = 0;
  // items per user and their exclusive scan (item_off[u] = first item of u)
  int64_t cnt = 0;
  for (int u = u0; u < u1; ++u) cnt += items_of(u);
  int64_t base, dummy, total, dummy2;
  block_exscan2(cnt, 0, &base, &dummy, &total, &dummy2);
  for (int u = u0; u < u1; ++u) {
    item_off[u] = (int32_t)base;
    if (off_smem) s_item_off[u] = (int32_t)base;
    base += items_of(u);
  }
  if (tid == 0) {
    item_off[B] = (int32_t)total;
    if (off_smem) s_item_off[B] = (int32_t)total;
  }
  __syncthreads();
  const int32_t* ioff = off_smem ? s_item_off : item_off;
  auto cost_of = [&](int u, int b) {
    const int64_t q = (int64_t)nl[u] + n_q;
    const int64_t jl = per_head ? min((int64_t)(b / heads) * 128 + 127, q - 1)
                                : min((int64_t)b * 128 + 127, q * heads - 1) / heads;
    const int64_t kmax = jl < nl[u] ? (int64_t)Tl[u] - nl[u] + jl + 1 : (int64_t)Tl[u];
    const int64_t tiles = (kmax + attn_keys - 1) / attn_keys;
    return (int)(tiles < kBuckets - 1 ? tiles : kBuckets - 1);
  };
  auto user_of = [&](int i) {      // largest u with item_off[u] <= i
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ioff[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  int32_t* W = p.work + (int64_t)l * 2 * p.max_work;
  if (per_head) {
    // users by the key tiles of their last row (bucketed, descending); each
    // user claims one consecutive range of the list for its items
    auto ucost = [&](int u) {
      const int64_t tiles = ((int64_t)Tl[u] + attn_keys - 1) / attn_keys;
      return (int)(tiles < kBuckets - 1 ? tiles : kBuckets - 1);
    };
    for (int u = u0; u < u1; ++u) atomicAdd(&hist[ucost(u)], (int32_t)items_of(u));
    __syncthreads();
    if (tid == 0) {
      int32_t acc = 0;
      for (int k = kBuckets - 1; k >= 0; --k) { cursor[k] = acc; acc += hist[k]; }
      total_items = acc;
    }
    __syncthreads();
    for (int u = u0; u < u1; ++u) {
      const int32_t n_items_u = (int32_t)items_of(u);
      if (n_items_u == 0) continue;
      const int32_t nblk = n_items_u / heads;
      const int32_t ubase = atomicAdd(&cursor[ucost(u)], n_items_u);
      for (int32_t b = 0; b < n_items_u; ++b) {
        const int32_t blk = b / heads, head = b % heads;
        const int32_t pos = ubase + head * nblk + (nblk - 1 - blk);
        W[2 * pos] = u;
        W[2 * pos + 1] = b;
      }
    }
    if (tid == 0) {
      p.work_count[l] = total_items;
      p.work_next[l] = 0;
    }
    return;
  }
  for (int i = tid; i < (int)total; i += kPlanThreads) {
    const int u = user_of(i);
    atomicAdd(&hist[cost_of(u, i - ioff[u])], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int32_t acc = 0;
    for (int k = kBuckets - 1; k >= 0; --k) { cursor[k] = acc; acc += hist[k]; }
    total_items = acc;
  }
  __syncthreads();
  for (int i = tid; i < (int)total; i += kPlanThreads) {
    const int u = user_of(i);
    const int b = i - ioff[u];
    const int pos = atomicAdd(&cursor[cost_of(u, b)], 1);
    W[2 * pos] = u;
    W[2 * pos + 1] = b;
  }
  if (tid == 0) {
    p.work_count[l] = total_items;
    p.work_next[l] = 0;
  }
}

cudaError_t launch_plan(const llatte_handle* h, const int64_t* offsets, int B, cudaStream_t s) {
  KeepArr k;
  const int L = h->dims.n_layers;
  for (int i = 0; i <= LLATTE_MAX_LAYERS; ++i) k.k[i] = i < L ? h->dims.keep[i] : 0;
  plan_kernel<<<L + 1, kPlanThreads, 0, s>>>(offsets, B, h->plan, k, L, h->dims.n_q, h->dims.max_len,
                                          h->max_rows_h, h->dims.heads, h->use_tc ? h->attn_keys : 0,
                                          h->heads_mask);
  return cudaGetLastError();
}

cudaError_t launch_plan_on(const PlanDev& p, const llatte_dims& d, int64_t max_total,
                           const int64_t* offsets, int B, cudaStream_t s) {
  KeepArr k;
  for (int i = 0; i <= LLATTE_MAX_LAYERS; ++i) k.k[i] = i < d.n_layers ? d.keep[i] : 0;
  plan_kernel<<<d.n_layers + 1, kPlanThreads, 0, s>>>(offsets, B, p, k, d.n_layers, d.n_q, d.max_len,
                                          max_total, d.heads, 0, 0u);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- gather

// sin and cos of x: x is reduced to [-pi, pi] by subtracting the nearest
// multiple of 2 pi in two parts (Cody and Waite's method; 2 pi = 6.28125 +
// a remainder, the first part short enough that k * 6.28125 is exact for
// |k| < 2^16, i.e. |x| < 4e5), then the hardware approximation, whose absolute
// error is below 1e-6 on that interval.
__device__ __forceinline__ void sincos_reduced(float x, float* s, float* c) {
  constexpr float kInv2Pi = 0.15915494309189535f;
  constexpr float kHi = 6.28125f, kLo = 1.9353071795864769e-3f;
  const float k = rintf(x * kInv2Pi);
  float r = fmaf(-k, kHi, x);
  r = fmaf(-k, kLo, r);
  __sincosf(r, s, c);
}

// Additive timestamp code (LLaTTE notes, appendix A.2 item 1, read as the
// Transformer's sinusoidal code of the event's age in hours): the 16-byte
// vector x holds dims e0 .. e0 + 16/elem - 1 of a history row; dims 2i and
// 2i + 1 below d_time add sin(age w_i) and cos(age w_i), w_i = 10000^(-2i/d_time).
__device__ __forceinline__ void add_time_code(uint4& x, int e0, float age, int d_time, int elem) {
  constexpr float kLog2Base = 13.287712379549449f;       // log2(10000)
  if (elem == 2) {
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = e0 + 2 * k;                            // even: one (sin, cos) pair
      if (e >= d_time) break;
      float sn, cs;
      sincos_reduced(age * exp2f(-(float)e / (float)d_time * kLog2Base), &sn, &cs);
      float2 f = __bfloat1622float2(h2[k]);
      f.x += sn;
      f.y += cs;
      h2[k] = __floats2bfloat162_rn(f.x, f.y);
    }
  } else {
    float* f = reinterpret_cast<float*>(&x);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = e0 + 2 * k;
      if (e >= d_time) break;
      float sn, cs;
      sincos_reduced(age * exp2f(-(float)e / (float)d_time * kLog2Base), &sn, &cs);
      f[2 * k] += sn;
      f[2 * k + 1] += cs;
    }
  }
}

// Block (u, s): slice s of user u's rows.  Rows 0..T-1 are the user's
// history events, each read once and stored to the history buffer and, for
// the last n, also to the query rows; rows T..T+n_q-1 are the query tokens
// (query rows n..).  One warp per row.  With ages, every history event gets
// the timestamp code.
__global__ void __launch_bounds__(256)
gather_kernel(const uint4* __restrict__ values, const int64_t* __restrict__ offsets,
              const uint4* __restrict__ cand, PlanDev p, uint4* __restrict__ Xh,
              uint4* __restrict__ Xq, int row_vecs, int n_q, int n_layers,
              const float* __restrict__ ages, int d_time, int elem) {
  // a batch the plan rejected has zero rows everywhere: copy nothing
  if (*p.hist_total(0) == 0 && *p.query_total(0) == 0) return;
  const int u = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int warps = (blockDim.x >> 5) * gridDim.y;
  const int w0 = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t T = p.Tl(0)[u], n = p.nl(0)[u];
  const int64_t hoff = p.hoff(0)[u], qoff = p.qoff(0)[u], src0 = offsets[u];
  const int64_t rows = T + n_q;
  // user of every query row of every layer (the epilogues' row -> user map)
  for (int l = 0; l < n_layers; ++l) {
    const int64_t q = (int64_t)p.nl(l)[u] + n_q;
    int32_t* dst = p.row_user + l * p.row_user_stride + p.qoff(l)[u];
    for (int64_t j = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; j < q;
         j += (int64_t)gridDim.y * blockDim.x)
      dst[j] = u;
  }
  // four rows in flight per warp: all loads of a group before its stores
  constexpr int RG = 4;
  for (int64_t r0 = w0; r0 < rows; r0 += (int64_t)warps * RG) {
    const uint4* src[RG];
    uint4* dst[RG];
    uint4* dst2[RG];                     // kept history rows: also a query row
    float age[RG];                       // -1: no timestamp code (query token / none)
#pragma unroll
    for (int k = 0; k < RG; ++k) {
      const int64_t r = r0 + (int64_t)k * warps;
      src[k] = nullptr;
      dst[k] = nullptr;
      dst2[k] = nullptr;
      age[k] = -1.f;
      if (r >= rows) continue;
      if (r < T) {
        src[k] = values + (src0 + r) * row_vecs;
        dst[k] = Xh + (hoff + r) * row_vecs;
        if (r >= T - n) dst2[k] = Xq + (qoff + r - (T - n)) * row_vecs;
        if (ages) age[k] = __ldg(ages + src0 + r);
      } else {
        const int64_t j = r - T;
        src[k] = cand + ((int64_t)u * n_q + j) * row_vecs;
        dst[k] = Xq + (qoff + n + j) * row_vecs;
      }
    }
    const int epv = 16 / elem;           // elements per 16-byte vector
    for (int v = lane; v < row_vecs; v += 32) {
      uint4 x[RG];
#pragma unroll
      for (int k = 0; k < RG; ++k)
        if (src[k]) x[k] = __ldg(src[k] + v);
      if (ages && v * epv < d_time) {
#pragma unroll
        for (int k = 0; k < RG; ++k)
          if (src[k] && age[k] >= 0.f) add_time_code(x[k], v * epv, age[k], d_time, elem);
      }
#pragma unroll
      for (int k = 0; k < RG; ++k) {
        if (dst[k]) dst[k][v] = x[k];
        if (dst2[k]) dst2[k][v] = x[k];
      }
    }
  }
}

cudaError_t launch_gather(const llatte_handle* h, const void* values, const int64_t* offsets,
                          const void* cand, const float* ages, int B, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const int row_vecs = h->dims.d * h->elem / 16;
  // enough blocks to cover every SM several times even for small batches
  const int slices = std::max(1, std::min(64, (h->num_sms * 8 + B - 1) / B));
  gather_kernel<<<dim3(B, slices), 256, 0, s>>>((const uint4*)values, offsets, (const uint4*)cand,
                                                h->plan, (uint4*)h->Xh[0], (uint4*)h->Xq[0],
                                                row_vecs, h->dims.n_q, h->dims.n_layers,
                                                h->dims.d_time > 0 ? ages : nullptr,
                                                h->dims.d_time, h->elem);
  return cudaGetLastError();
}

}  // namespace llatte
