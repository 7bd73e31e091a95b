// Host runtime of the LLaTTE forward library: argument checks, weight
// absorption, workspace, the per-layer launch sequence and per-step timing.
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <new>

#include "internal.h"
#include "tc_attn.h"
#include "tc_ffn.h"
#include "tc_gemm.h"

using namespace llatte;

namespace llatte {
const char* const kStepNames[ST_COUNT] = {"plan", "gather", "ctx_bias", "kv",      "q",  "attn",
                                          "o",    "ffn1",   "ffn2",     "readout", "ffn",
                                          "summary", "attn_export"};
}

namespace {

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

// Split-K of the summary bottleneck GEMM: about this many CTAs in all (the
// SM count of a B200); the workspace bound below follows from it.
constexpr int kSplitCtas = 148;
constexpr int kSumMaxBN = 128;

int summary_slices(int64_t B, int N, int BN, int K) {
  const int64_t tiles = ((B + 127) / 128) * (N / BN);
  const int64_t KB = K / 64;
  return (int)std::max<int64_t>(1, std::min<int64_t>(KB, kSplitCtas / std::max<int64_t>(tiles, 1)));
}

struct Layout {
  int64_t rows_h, rows_q;
  size_t off_hist_off, off_query_off, off_T, off_n, off_totals, off_status, off_work,
      off_work_count, off_work_next, off_item_off, off_row_user;
  size_t off_Xh[2], off_Xq[2], off_C, off_Qt, off_Ot, off_Z, off_Hd, off_Cq, off_acc32, off_ctxbias,
      off_final, off_mean, off_mean16, off_Zres, off_Xqres[2], off_zraw, off_sum_part, off_sum_h,
      off_sum_h16, off_KV;
  size_t total;
  int32_t max_work;
};

uint32_t heads_mask_of(const llatte_dims& D);

int check_dims(const llatte_dims* d) {
  if (!d) return LLATTE_ERR_ARG;
  if (d->n_layers < 1 || d->n_layers > LLATTE_MAX_LAYERS) return LLATTE_ERR_ARG;
  if (d->d <= 0 || d->heads <= 0 || d->d_head <= 0 || d->rank <= 0) return LLATTE_ERR_ARG;
  if (d->d_ctx < 0 || d->n_q < 0 || d->d_out < 0 || d->ffn_mult <= 0) return LLATTE_ERR_ARG;
  if (d->dtype != LLATTE_BF16 && d->dtype != LLATTE_FP32) return LLATTE_ERR_ARG;
  if (!(d->eps > 0.f)) return LLATTE_ERR_ARG;
  if (d->max_batch <= 0 || d->max_len < 0 || d->max_total < 0) return LLATTE_ERR_ARG;
  if (d->kv_norm != 0 && d->kv_norm != 1) return LLATTE_ERR_ARG;
  if (d->n_sum < 0 || d->n_sum > LLATTE_MAX_SUMMARIES) return LLATTE_ERR_ARG;
  if (d->q_rank < 0) return LLATTE_ERR_ARG;
  if (d->d_time < 0 || d->d_time % 2 != 0 || d->d_time > d->d) return LLATTE_ERR_ARG;
  if (d->attn_form < LLATTE_ATTN_AUTO || d->attn_form > LLATTE_ATTN_PER_HEAD) return LLATTE_ERR_ARG;
  if (d->q_rank > 1024) return LLATTE_ERR_UNSUPPORTED;
  if (d->n_sum > 0) {
    if (d->n_q <= 0 || d->d_out > 0 || d->sum_rank <= 0 || d->d_seq <= 0) return LLATTE_ERR_ARG;
    if (d->sum_rank > 1024 || d->d_seq % 2 != 0) return LLATTE_ERR_UNSUPPORTED;
  }
  for (int l = 0; l < d->n_layers; ++l) {
    if (d->keep[l] < 0) return LLATTE_ERR_ARG;
    if (l && d->keep[l] > d->keep[l - 1]) return LLATTE_ERR_ARG;  // T_{l+1} <= T_l
  }
  const int elem = d->dtype == LLATTE_BF16 ? 2 : 4;
  if ((d->d * elem) % 16 != 0) return LLATTE_ERR_UNSUPPORTED;     // 16-byte row vectors
  if (d->rank > 256) return LLATTE_ERR_UNSUPPORTED;
  if (d->attn_form == LLATTE_ATTN_PER_HEAD && heads_mask_of(*d) == 0) return LLATTE_ERR_UNSUPPORTED;
  return LLATTE_OK;
}

Layout layout_of(const llatte_dims* d) {
  Layout L;
  const int elem = d->dtype == LLATTE_BF16 ? 2 : 4;
  const int64_t B = d->max_batch;
  L.rows_h = d->max_total ? d->max_total : B * d->max_len;
  L.rows_q = std::min<int64_t>(L.rows_h, B * (int64_t)d->keep[0]) + B * d->n_q;
  const int64_t hr = (int64_t)d->heads * d->rank, f = (int64_t)d->ffn_mult * d->d;
  const int nl = d->n_layers;
  // attention work items: (user, 128-row block of (query row, head) pairs)
  // (absorbed: blocks of 128 (row, head) pairs; per-head: h blocks per 128 rows)
  const int64_t max_work = (L.rows_q * d->heads + 127) / 128 + B * d->heads;
  L.max_work = (int32_t)std::min<int64_t>(max_work, 1 << 30);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o += align_up(bytes); return r; };
  L.off_hist_off = take(sizeof(int64_t) * (nl + 1) * (B + 1));
  L.off_query_off = take(sizeof(int64_t) * (nl + 1) * (B + 1));
  L.off_T = take(sizeof(int32_t) * (nl + 1) * B);
  L.off_n = take(sizeof(int32_t) * (nl + 1) * B);
  L.off_totals = take(sizeof(int64_t) * 2 * (nl + 1));
  L.off_status = take(sizeof(int32_t));
  L.off_work = take(sizeof(int32_t) * 2 * nl * (size_t)L.max_work);
  L.off_work_count = take(sizeof(int32_t) * nl);
  L.off_work_next = take(sizeof(int32_t) * nl);
  L.off_item_off = take(sizeof(int32_t) * (B + 1) * nl);     // per layer
  L.off_row_user = take(sizeof(int32_t) * nl * (size_t)L.rows_q);
  for (int i = 0; i < 2; ++i) L.off_Xh[i] = take((size_t)L.rows_h * d->d * elem);
  for (int i = 0; i < 2; ++i) L.off_Xq[i] = take((size_t)L.rows_q * d->d * elem);
  L.off_C = take((size_t)L.rows_h * d->rank * elem);
  L.off_Qt = take((size_t)L.rows_q * hr * elem);
  L.off_Ot = take((size_t)L.rows_q * hr * elem);
  L.off_Z = take((size_t)L.rows_q * d->d * elem);
  L.off_Hd = take((size_t)L.rows_q * f * elem);
  L.off_Cq = take((size_t)L.rows_q * d->q_rank * elem);
  const int64_t hdh = (int64_t)d->heads * d->d_head;
  L.off_KV = take(heads_mask_of(*d) ? (size_t)L.rows_h * 2 * hdh * elem : 0);
  // fp16 copies of the residual stream (bf16 storage keeps bf16 GEMM operands
  // plus these; fp32 storage needs none)
  const size_t res16 = elem == 2 ? 2 * (size_t)L.rows_q * d->d : 0;
  L.off_Zres = take(res16);
  for (int i = 0; i < 2; ++i) L.off_Xqres[i] = take(res16);
  L.off_acc32 = take(sizeof(float) * std::max<size_t>(
                                         std::max<size_t>((size_t)L.rows_h * d->rank,
                                                          (size_t)L.rows_q * d->d),
                                         (size_t)L.rows_q * d->q_rank));
  // per-user context term of every layer's query: h*r columns (full-rank
  // query), or q_rank columns (low-rank query: it enters before the norm)
  L.off_ctxbias = take(sizeof(float) * nl * B *
                       std::max<int64_t>(std::max<int64_t>(hr, d->q_rank), hdh));
  L.off_final = take(d->d_out ? sizeof(float) * L.rows_q * d->d : 0);
  L.off_mean = take(d->d_out ? sizeof(float) * B * d->d : 0);
  L.off_mean16 = take(d->d_out && elem == 2 ? 2 * (size_t)B * d->d : 0);
  // sequence summaries: the final query-token rows and the split-K partials
  // (S * B <= kSplitCtas * 128 / column tiles, or S = 1)
  const int64_t sN = (int64_t)d->n_sum * d->sum_rank;
  L.off_zraw = take(d->n_sum ? (size_t)B * d->n_q * d->d * elem : 0);
  L.off_sum_part = take(d->n_sum ? sizeof(float) * std::max<int64_t>(
                                       (int64_t)kSplitCtas * 128 * kSumMaxBN, B * sN) : 0);
  L.off_sum_h = take(d->n_sum ? sizeof(float) * B * sN : 0);
  L.off_sum_h16 = take(d->n_sum ? 2 * (size_t)((B + 127) / 128 * 128) * sN : 0);
  L.total = o;
  return L;
}

#define CK(x)                                                   \
  do {                                                          \
    cudaError_t e_ = (x);                                       \
    if (e_ != cudaSuccess) {                                    \
      fprintf(stderr, "llatte: %s failed: %s (%s:%d)\n", #x,    \
              cudaGetErrorString(e_), __FILE__, __LINE__);      \
      return LLATTE_ERR_CUDA;                                   \
    }                                                           \
  } while (0)

void* dev_alloc(llatte_handle* h, size_t bytes) {
  void* p = nullptr;
  if (cudaMalloc(&p, bytes ? bytes : 16) != cudaSuccess) return nullptr;
  h->allocs.push_back(p);
  return p;
}

// Copy one weight array to a fresh device buffer.
void* upload(llatte_handle* h, const void* src, size_t bytes, int on_device) {
  void* p = dev_alloc(h, bytes);
  if (!p) return nullptr;
  if (bytes && cudaMemcpy(p, src, bytes, on_device ? cudaMemcpyDeviceToDevice
                                                    : cudaMemcpyHostToDevice) != cudaSuccess)
    return nullptr;
  return p;
}

cudaEvent_t take_event(llatte_handle* h) {
  if (!h->event_pool.empty()) {
    cudaEvent_t e = h->event_pool.back();
    h->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct StepTimer {
  llatte_handle* h;
  cudaStream_t s;
  int step;
  cudaEvent_t a = nullptr;
  StepTimer(llatte_handle* h_, cudaStream_t s_, int step_) : h(h_), s(s_), step(step_) {
    if (h->profiling) {
      a = take_event(h);
      cudaEventRecord(a, s);
    }
  }
  // Records the step's end once; the start event then belongs to the record
  // (a second call would put one event into two records).
  void done(int launches) {
    if (!h->profiling || !a) return;
    cudaEvent_t b = take_event(h);
    cudaEventRecord(b, s);
    h->pending.push_back(ProfRec{step, a, b, launches});
    a = nullptr;
  }
  // A step left early (an error return) hands its start event back.
  ~StepTimer() {
    if (a) h->event_pool.push_back(a);
  }
};

int drain_profile(llatte_handle* h) {
  for (auto& r : h->pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return LLATTE_ERR_CUDA;
    cudaEventElapsedTime(&ms, r.a, r.b);
    h->step_ms[r.step] += ms;
    h->step_launches[r.step] += r.launches;
    h->step_calls[r.step] += 1;
    h->event_pool.push_back(r.a);
    h->event_pool.push_back(r.b);
  }
  h->pending.clear();
  return LLATTE_OK;
}


// Dimensions the tensor-core kernels implement (bf16 storage).
bool tc_dims_ok(const llatte_dims& D) {
  const int hr = D.heads * D.rank, f = D.ffn_mult * D.d;
  const bool d_ok = D.d == 64 || D.d == 128 || D.d == 256 || D.d == 512;
  const bool r_ok = attn_tc_supported(D.rank);
  // low-rank query: its latent is normalised in one 128 x q_rank tile
  const bool q_ok = D.q_rank == 0 || D.q_rank == 64 || D.q_rank == 128 || D.q_rank == 256 ||
                    D.q_rank == 512;
  return d_ok && r_ok && q_ok && hr % 64 == 0 && f % 64 == 0;
}

// Layers that run MLA in its per-head form (K, V = split(c_kv W_up^KV),
// scores over d_h = 64).  Both forms compute the same function; per layer the
// per-head one does 4 d_h / (4 r) of the absorbed attention's tensor work and
// smaller query / output projections, at the price of one up-projection of
// the keys, so "auto" takes it when r > 2 d_h.
uint32_t heads_mask_of(const llatte_dims& D) {
  const bool possible = D.dtype == LLATTE_BF16 && tc_dims_ok(D) && D.d_head == 64 &&
                        D.q_rank == 0;
  if (!possible || D.attn_form == LLATTE_ATTN_ABSORBED) return 0;
  if (D.attn_form == LLATTE_ATTN_AUTO && D.rank <= 2 * D.d_head) return 0;
  return D.n_layers >= 32 ? 0xffffffffu : ((1u << D.n_layers) - 1);
}

int pick_bn(int N) { return N % 256 == 0 ? 256 : N % 128 == 0 ? 128 : 64; }

bool build_tc_maps(llatte_handle* h) {
  const llatte_dims& D = h->dims;
  const int d = D.d, r = D.rank, hr = D.heads * D.rank, f = D.ffn_mult * D.d;
  h->bn_kv = r;
  h->bn_q = pick_bn(hr);
  h->bn_o = d;
  h->bn_f1 = pick_bn(f);
  h->bn_f2 = d;
  h->bn_dq = D.q_rank;
  const int kq = D.q_rank ? D.q_rank : d;     // input width of the absorbed query GEMM
  const uint64_t rh = std::max<int64_t>(h->max_rows_h, 1), rq = std::max<int64_t>(h->max_rows_q, 1);
  bool ok = true;
  for (int i = 0; i < 2; ++i) {
    ok = ok && make_tmap_bf16(&h->tm_Xh[i], h->Xh[i], rh, d, 128);
    ok = ok && make_tmap_bf16(&h->tm_Xq[i], h->Xq[i], rq, d, 128);
  }
  ok = ok && make_tmap_bf16(&h->tm_Ot, h->Ot, rq, hr, 128);
  ok = ok && make_tmap_bf16(&h->tm_Z, h->Z, rq, d, 128);
  if (h->Zres) ok = ok && make_tmap_f16(&h->tm_Zres, h->Zres, rq, d, 128);
  for (int i = 0; i < 2 && h->Xqres[i]; ++i)
    ok = ok && make_tmap_f16(&h->tm_Xqres[i], h->Xqres[i], rq, d, 128);
  ok = ok && make_tmap_bf16(&h->tm_Hd, h->Hd, rq, f, 128);
  if (D.q_rank) ok = ok && make_tmap_bf16(&h->tm_Cq, h->Cq, rq, D.q_rank, 128);
  h->attn_keys = attn_tc_keys(r);
  h->ffn_fused = ffn_tc_supported(d, f) ? 1 : 0;
  h->pair_norm = tc_gemm_pair_supported(TC_NORM, d, hr) && tc_gemm_pair_supported(TC_NORM, d, f);
  ok = ok && make_tmap_bf16(&h->tm_Qt, h->Qt, rq * D.heads, r, 128);
  ok = ok && make_tmap_bf16(&h->tm_C, h->C, rh, r, (uint32_t)h->attn_keys);
  const int hdh = D.heads * D.d_head;
  if (h->heads_mask) {
    ok = ok && make_tmap_bf16(&h->tm_Qh, h->Qt, rq, hdh, 128);
    ok = ok && make_tmap_bf16(&h->tm_KV, h->KV, rh, 2 * hdh, 128);
    ok = ok && make_tmap_bf16(&h->tm_Oh, h->Ot, rq, hdh, 128);
    h->pair_norm = h->pair_norm && tc_gemm_pair_supported(TC_NORM, d, hdh);
  }
  // readout projection: [max_batch, d] bf16 means times E^T, 64-column tiles
  h->readout_tc = D.d_out > 0 && h->mean16 && D.d_out % 64 == 0 ? 1 : 0;
  if (h->readout_tc) {
    ok = ok && make_tmap_bf16(&h->tm_mean16, h->mean16, std::max(D.max_batch, 1), d, 128);
    ok = ok && make_tmap_bf16(&h->tm_We, h->W_e, D.d_out, d, 64);
  }
  ok = ok && make_tmap_store16(&h->tms_C, h->C, rh, r, false);
  ok = ok && make_tmap_store16(&h->tms_Qt, h->Qt, rq, hr, false);
  ok = ok && make_tmap_store16(&h->tms_Hd, h->Hd, rq, f, false);
  if (h->Zres) ok = ok && make_tmap_store16(&h->tms_Zres, h->Zres, rq, d, true);
  if (D.q_rank) ok = ok && make_tmap_store16(&h->tms_Cq, h->Cq, rq, D.q_rank, false);
  if (h->heads_mask) {
    ok = ok && make_tmap_store16(&h->tms_KV, h->KV, rh, 2 * hdh, false);
    ok = ok && make_tmap_store16(&h->tms_Qh, h->Qt, rq, hdh, false);
  }
  // weight tiles load in boxes of at most 128 rows (an SM pair's CTA loads
  // one 128-row half of a 256-row tile; the one-SM kernel stacks boxes)
  auto box = [](int bn) { return (uint32_t)std::min(bn, 128); };
  for (int l = 0; l < D.n_layers && ok; ++l) {
    const LayerDev& W = h->layers[l];
    LayerMaps& M = h->lmaps[l];
    ok = ok && make_tmap_bf16(&M.dkv, W.W_dkv, r, d, box(h->bn_kv));
    ok = ok && make_tmap_bf16(&M.qk, W.W_qk, hr, kq, box(h->bn_q));
    if (D.q_rank) ok = ok && make_tmap_bf16(&M.dq, W.W_dqx, D.q_rank, d, box(h->bn_dq));
    if ((h->heads_mask >> l) & 1u) {
      ok = ok && make_tmap_bf16(&M.qh, W.W_qh, hdh, d, box(pick_bn(hdh)));
      ok = ok && make_tmap_bf16(&M.ukv, W.W_ukv, 2 * hdh, r, box(pick_bn(2 * hdh)));
      ok = ok && make_tmap_bf16(&M.oh, W.W_oh, d, hdh, box(h->bn_o));
      if (h->pair_norm) ok = ok && make_tmap_bf16(&M.oh_pair, W.W_oh, d, hdh, 128);
    }
    ok = ok && make_tmap_bf16(&M.ov, W.W_ov, d, hr, box(h->bn_o));
    ok = ok && make_tmap_bf16(&M.w1, W.W1, f, d, box(h->bn_f1));
    ok = ok && make_tmap_bf16(&M.w2, W.W2, d, f, box(h->bn_f2));
    // layers >= 1 with a full-rank query read their query rows in fp16 (the
    // residual copy), so their query weight gets an fp16 copy
    if (l >= 1 && !D.q_rank && h->Xqres[0]) {
      LayerDev& Wm = h->layers[l];
      const bool ph = (h->heads_mask >> l) & 1u;
      const int rows = ph ? hdh : hr;
      if (ok && !Wm.W_q16) {
        Wm.W_q16 = dev_alloc(h, 2 * (size_t)rows * d);
        ok = Wm.W_q16 && launch_bf16_to_f16(ph ? W.W_qh : W.W_qk, Wm.W_q16, (int64_t)rows * d, 0) ==
                             cudaSuccess;
      }
      if (ph) ok = ok && make_tmap_f16(&M.qh16, Wm.W_q16, hdh, d, box(pick_bn(hdh)));
      else ok = ok && make_tmap_f16(&M.qk16, Wm.W_q16, hr, d, box(h->bn_q));
    }
    // the FFN's first product takes Z in fp16 (the residual copy, so Z crosses
    // HBM once), so W1 gets an fp16 copy (both operands of an MMA share a type)
    {
      LayerDev& Wm = h->layers[l];
      if (ok && !Wm.W1h) {
        Wm.W1h = dev_alloc(h, 2 * (size_t)f * d);
        ok = Wm.W1h && launch_bf16_to_f16(W.W1, Wm.W1h, (int64_t)f * d, 0) == cudaSuccess;
      }
      ok = ok && make_tmap_f16(&M.w1h, Wm.W1h, f, d, box(h->bn_f1));
      if (h->ffn_fused) {
        // the SM-pair FFN: each CTA loads half of a weight chunk
        ok = ok && make_tmap_bf16(&M.w1_pair, W.W1, f, d, 64);
        ok = ok && make_tmap_bf16(&M.w2_pair, W.W2, d, f, 128);
        ok = ok && make_tmap_f16(&M.w1h_pair, Wm.W1h, f, d, 64);
      }
    }
    if (h->pair_norm) {
      // the SM-pair residual + RMSNorm GEMMs at d = 512: 128-row weight boxes
      ok = ok && make_tmap_bf16(&M.ov_pair, W.W_ov, d, hr, 128);
      ok = ok && make_tmap_bf16(&M.w2_pair, W.W2, d, f, 128);
    }
  }
  return ok;
}

}  // namespace

extern "C" {

size_t llatte_workspace_bytes(const llatte_dims* dims) {
  if (check_dims(dims) != LLATTE_OK) return 0;
  return layout_of(dims).total;
}

const char* llatte_error_string(int code) {
  switch (code) {
    case LLATTE_OK: return "ok";
    case LLATTE_ERR_ARG: return "invalid argument";
    case LLATTE_ERR_UNSUPPORTED: return "unsupported dimensions";
    case LLATTE_ERR_CUDA: return "CUDA runtime error";
    case LLATTE_ERR_OOM: return "device allocation failed";
    case LLATTE_ERR_DEVICE: return "device-side fault reported in the status word";
    default: return "unknown error";
  }
}

void llatte_destroy(llatte_handle* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  if (h->side) cudaStreamDestroy(h->side);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  for (auto& r : h->pending) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
  for (auto e : h->event_pool) cudaEventDestroy(e);
  for (void* p : h->allocs) cudaFree(p);
  delete h;
}

int llatte_create(llatte_handle** out, const llatte_dims* dims, const llatte_layer_w* layers,
                  const void* W_e, const llatte_summary_w* summaries, int weights_on_device) {
  if (!out) return LLATTE_ERR_ARG;
  *out = nullptr;
  int rc = check_dims(dims);
  if (rc != LLATTE_OK) return rc;
  if (!layers) return LLATTE_ERR_ARG;
  const llatte_dims& D = *dims;
  for (int l = 0; l < D.n_layers; ++l) {
    const llatte_layer_w& w = layers[l];
    if (!w.W_dkv || !w.g_kv || !w.W_uk || !w.W_uv || !w.W_o || !w.g1 || !w.W1 || !w.W2 || !w.g2)
      return LLATTE_ERR_ARG;
    if (D.q_rank ? (!w.W_dq || !w.g_q || !w.W_uq) : !w.W_q) return LLATTE_ERR_ARG;
  }
  if (D.d_out > 0 && !W_e) return LLATTE_ERR_ARG;
  if (D.n_sum > 0) {
    if (!summaries) return LLATTE_ERR_ARG;
    for (int k = 0; k < D.n_sum; ++k)
      if (!summaries[k].W_down || !summaries[k].W_up) return LLATTE_ERR_ARG;
  }

  llatte_handle* h = new (std::nothrow) llatte_handle();
  if (!h) return LLATTE_ERR_OOM;
  h->dims = D;
  h->elem = D.dtype == LLATTE_BF16 ? 2 : 4;
  h->use_tc = 0;
  h->inject_timeout = 0;
  h->profiling = 0;
  h->last_B = 0;
  h->export_req = nullptr;
  for (int i = 0; i < ST_COUNT; ++i) { h->step_ms[i] = 0; h->step_launches[i] = 0; h->step_calls[i] = 0; }
  auto fail = [&](int code) { llatte_destroy(h); return code; };
  if (cudaGetDevice(&h->device) != cudaSuccess) return fail(LLATTE_ERR_CUDA);
  if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess)
    return fail(LLATTE_ERR_CUDA);
  if (cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess)
    return fail(LLATTE_ERR_CUDA);

  const size_t e = h->elem;
  const int d = D.d, r = D.rank, hd = D.heads * D.d_head, hr = D.heads * D.rank,
            f = D.ffn_mult * D.d, dc = D.d_ctx, rq = D.q_rank;
  // columns of the matrix absorbed into the query: W_q [hd, d + dc], or for a
  // low-rank query W_uq [hd, rq] (the context then enters through W_dq)
  const int kq = rq ? rq : d, kqc = rq ? 0 : dc;
  // The tensor-core attention takes its scores in log2 units (exp2 in the
  // softmax): fold log2(e) into the absorbed query projection for that path.
  const bool want_tc = h->elem == 2 && tc_dims_ok(D);
  const uint32_t heads_mask = want_tc ? heads_mask_of(D) : 0u;
  h->heads_mask = heads_mask;
  const float qscale = want_tc ? 1.4426950408889634f : 1.0f;
  for (int l = 0; l < D.n_layers; ++l) {
    const llatte_layer_w& w = layers[l];
    LayerDev& L = h->layers[l];
    L.W_dkv = upload(h, w.W_dkv, e * r * d, weights_on_device);
    L.g_kv = upload(h, w.g_kv, e * r, weights_on_device);
    L.g1 = upload(h, w.g1, e * d, weights_on_device);
    L.W1 = upload(h, w.W1, e * (size_t)f * d, weights_on_device);
    L.W2 = upload(h, w.W2, e * (size_t)d * f, weights_on_device);
    L.g2 = upload(h, w.g2, e * d, weights_on_device);
    L.W_qk = dev_alloc(h, e * (size_t)hr * kq);
    L.W_qkc = kqc ? (float*)dev_alloc(h, sizeof(float) * (size_t)hr * kqc) : nullptr;
    L.W_ov = dev_alloc(h, e * (size_t)d * hr);
    L.W_dqx = L.g_q = nullptr;
    L.W_dqc = nullptr;
    if (rq) {
      L.g_q = upload(h, w.g_q, e * rq, weights_on_device);
      L.W_dqx = dev_alloc(h, e * (size_t)rq * d);
      L.W_dqc = dc ? (float*)dev_alloc(h, sizeof(float) * (size_t)dc * rq) : nullptr;
      if (!L.g_q || !L.W_dqx || (dc && !L.W_dqc)) return fail(LLATTE_ERR_OOM);
      void* tdq = nullptr;
      bool okq = cudaMalloc(&tdq, e * (size_t)rq * (d + dc)) == cudaSuccess &&
                 cudaMemcpy(tdq, w.W_dq, e * (size_t)rq * (d + dc),
                            weights_on_device ? cudaMemcpyDeviceToDevice
                                              : cudaMemcpyHostToDevice) == cudaSuccess &&
                 launch_split_ctx_cols(h->elem, tdq, rq, d, dc, L.W_dqx, L.W_dqc, 1.f, 0) ==
                     cudaSuccess &&
                 cudaDeviceSynchronize() == cudaSuccess;
      cudaFree(tdq);
      if (!okq) return fail(LLATTE_ERR_CUDA);
    }
    if (!L.W_dkv || !L.g_kv || !L.g1 || !L.W1 || !L.W2 || !L.g2 || !L.W_qk || !L.W_ov ||
        (kqc && !L.W_qkc))
      return fail(LLATTE_ERR_OOM);
    L.W_qh = L.W_ukv = L.W_oh = nullptr;
    L.W_qhc = nullptr;
    if ((heads_mask >> l) & 1u) {
      // per-head form: W_q scaled by log2(e) / sqrt(d_h) (scores in log2
      // units), split into x and context columns; [W_uk ; W_uv]; W_o
      L.W_qh = dev_alloc(h, e * (size_t)hd * d);
      L.W_qhc = dc ? (float*)dev_alloc(h, sizeof(float) * (size_t)dc * hd) : nullptr;
      L.W_ukv = dev_alloc(h, e * (size_t)2 * hd * r);
      L.W_oh = upload(h, w.W_o, e * (size_t)d * hd, weights_on_device);
      if (!L.W_qh || (dc && !L.W_qhc) || !L.W_ukv || !L.W_oh) return fail(LLATTE_ERR_OOM);
      void* tw = nullptr;
      const cudaMemcpyKind kk = weights_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
      bool okh = cudaMalloc(&tw, e * (size_t)hd * (d + dc)) == cudaSuccess &&
                 cudaMemcpy(tw, w.W_q, e * (size_t)hd * (d + dc), kk) == cudaSuccess &&
                 launch_split_ctx_cols(h->elem, tw, hd, d, dc, L.W_qh, L.W_qhc,
                                       1.4426950408889634f / sqrtf((float)D.d_head), 0) ==
                     cudaSuccess &&
                 cudaMemcpy(L.W_ukv, w.W_uk, e * (size_t)hd * r, kk) == cudaSuccess &&
                 cudaMemcpy((char*)L.W_ukv + e * (size_t)hd * r, w.W_uv, e * (size_t)hd * r, kk) ==
                     cudaSuccess &&
                 cudaDeviceSynchronize() == cudaSuccess;
      cudaFree(tw);
      if (!okh) return fail(LLATTE_ERR_CUDA);
    }
    // temporaries for absorption
    void *tq = nullptr, *tuk = nullptr, *tuv = nullptr, *to = nullptr;
    bool ok = cudaMalloc(&tq, e * (size_t)hd * (kq + kqc)) == cudaSuccess &&
              cudaMalloc(&tuk, e * (size_t)hd * r) == cudaSuccess &&
              cudaMalloc(&tuv, e * (size_t)hd * r) == cudaSuccess &&
              cudaMalloc(&to, e * (size_t)d * hd) == cudaSuccess;
    cudaMemcpyKind k = weights_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    ok = ok && cudaMemcpy(tq, rq ? w.W_uq : w.W_q, e * (size_t)hd * (kq + kqc), k) == cudaSuccess &&
         cudaMemcpy(tuk, w.W_uk, e * (size_t)hd * r, k) == cudaSuccess &&
         cudaMemcpy(tuv, w.W_uv, e * (size_t)hd * r, k) == cudaSuccess &&
         cudaMemcpy(to, w.W_o, e * (size_t)d * hd, k) == cudaSuccess;
    ok = ok && launch_absorb(h->elem, tq, tuk, tuv, to, d, kq, kqc, D.heads, D.d_head, r, qscale,
                             L.W_qk, L.W_qkc, L.W_ov, 0) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    cudaFree(tq); cudaFree(tuk); cudaFree(tuv); cudaFree(to);
    if (!ok) return fail(LLATTE_ERR_CUDA);
  }
  h->W_e = nullptr;
  if (D.d_out > 0) {
    h->W_e = upload(h, W_e, e * (size_t)D.d_out * d, weights_on_device);
    if (!h->W_e) return fail(LLATTE_ERR_OOM);
  }
  h->W_sdown = h->W_sup = nullptr;
  // output projections as one batched tensor-core GEMM (bf16, K = sum_rank and
  // N = d_seq in whole 64-wide blocks); otherwise on CUDA cores
  h->sum_up_tc = want_tc && D.n_sum > 0 && D.sum_rank % 64 == 0 && D.d_seq % 64 == 0;
  if (D.n_sum > 0) {
    // bottleneck projections stacked into one [n_sum * sum_rank, n_q * d]
    // matrix; output projections stacked as given ([n_sum * d_seq, sum_rank],
    // tensor cores) or each transposed to [sum_rank][d_seq] (CUDA cores)
    const size_t rs = D.sum_rank, K = (size_t)D.n_q * d, ds = D.d_seq;
    h->W_sdown = dev_alloc(h, e * D.n_sum * rs * K);
    h->W_sup = dev_alloc(h, e * D.n_sum * rs * ds);
    if (!h->W_sdown || !h->W_sup) return fail(LLATTE_ERR_OOM);
    void* tmp = nullptr;
    if (cudaMalloc(&tmp, e * rs * ds) != cudaSuccess) return fail(LLATTE_ERR_OOM);
    const cudaMemcpyKind k = weights_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    bool ok = true;
    for (int j = 0; j < D.n_sum && ok; ++j) {
      ok = cudaMemcpy((char*)h->W_sdown + e * j * rs * K, summaries[j].W_down, e * rs * K, k) ==
               cudaSuccess &&
           cudaMemcpy(tmp, summaries[j].W_up, e * rs * ds, k) == cudaSuccess;
      if (!ok) break;
      if (h->sum_up_tc)
        ok = cudaMemcpy((char*)h->W_sup + e * j * rs * ds, tmp, e * rs * ds,
                        cudaMemcpyDeviceToDevice) == cudaSuccess;
      else
        ok = launch_transpose(h->elem, tmp, (int64_t)ds, (int64_t)rs,
                              (char*)h->W_sup + e * j * rs * ds, 0) == cudaSuccess;
      ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    }
    cudaFree(tmp);
    if (!ok) return fail(LLATTE_ERR_CUDA);
  }

  Layout Lo = layout_of(&D);
  char* ws = (char*)dev_alloc(h, Lo.total);
  if (!ws) return fail(LLATTE_ERR_OOM);
  if (cudaMemset(ws, 0, Lo.total) != cudaSuccess) return fail(LLATTE_ERR_CUDA);
  h->ws_bytes = Lo.total;
  h->max_rows_h = Lo.rows_h;
  h->max_rows_q = Lo.rows_q;
  PlanDev& p = h->plan;
  p.hist_off = (int64_t*)(ws + Lo.off_hist_off);
  p.query_off = (int64_t*)(ws + Lo.off_query_off);
  p.T = (int32_t*)(ws + Lo.off_T);
  p.n = (int32_t*)(ws + Lo.off_n);
  p.totals = (int64_t*)(ws + Lo.off_totals);
  p.status = (int32_t*)(ws + Lo.off_status);
  p.work = (int32_t*)(ws + Lo.off_work);
  p.work_count = (int32_t*)(ws + Lo.off_work_count);
  p.work_next = (int32_t*)(ws + Lo.off_work_next);
  p.item_off = (int32_t*)(ws + Lo.off_item_off);
  p.row_user = (int32_t*)(ws + Lo.off_row_user);
  p.row_user_stride = Lo.rows_q;
  p.stride = D.max_batch + 1;
  p.max_work = Lo.max_work;
  for (int i = 0; i < 2; ++i) { h->Xh[i] = ws + Lo.off_Xh[i]; h->Xq[i] = ws + Lo.off_Xq[i]; }
  h->C = ws + Lo.off_C;
  h->Qt = ws + Lo.off_Qt;
  h->Ot = ws + Lo.off_Ot;
  h->Z = ws + Lo.off_Z;
  h->Hd = ws + Lo.off_Hd;
  h->Cq = rq ? (void*)(ws + Lo.off_Cq) : nullptr;
  h->KV = heads_mask ? (void*)(ws + Lo.off_KV) : nullptr;
  h->Zres = h->elem == 2 ? (void*)(ws + Lo.off_Zres) : nullptr;
  for (int i = 0; i < 2; ++i) h->Xqres[i] = h->elem == 2 ? (void*)(ws + Lo.off_Xqres[i]) : nullptr;
  h->acc32 = (float*)(ws + Lo.off_acc32);
  h->ctxbias = (float*)(ws + Lo.off_ctxbias);
  h->final_rows = D.d_out ? (float*)(ws + Lo.off_final) : nullptr;
  h->mean_rows = D.d_out ? (float*)(ws + Lo.off_mean) : nullptr;
  h->mean16 = D.d_out > 0 && D.dtype == LLATTE_BF16 ? (void*)(ws + Lo.off_mean16) : nullptr;
  h->zraw = D.n_sum ? (void*)(ws + Lo.off_zraw) : nullptr;
  h->sum_part = D.n_sum ? (float*)(ws + Lo.off_sum_part) : nullptr;
  h->sum_h = D.n_sum ? (float*)(ws + Lo.off_sum_h) : nullptr;
  h->sum_h16 = D.n_sum ? (void*)(ws + Lo.off_sum_h16) : nullptr;
  h->sum_bpad = ((int64_t)D.max_batch + 127) / 128 * 128;
  h->sum_tc = 0;
  h->sum_bn = 0;
  if (want_tc) {
    if (!build_tc_maps(h)) return fail(LLATTE_ERR_CUDA);
    h->use_tc = 1;
    if (D.n_sum > 0) {
      const int N = D.n_sum * D.sum_rank, K = D.n_q * d;
      h->sum_bn = N % 128 == 0 ? 128 : 64;
      if (tc_gemm_supported(h->sum_bn, TC_F32, N, K)) {
        if (!make_tmap_bf16(&h->tm_zraw, h->zraw, D.max_batch, K, 128) ||
            !make_tmap_bf16(&h->tm_sdown, h->W_sdown, N, K, h->sum_bn))
          return fail(LLATTE_ERR_CUDA);
        h->sum_tc = 1;
      }
      if (h->sum_up_tc &&
          (!make_tmap_bf16(&h->tm_sh16, h->sum_h16, (uint64_t)D.n_sum * h->sum_bpad, D.sum_rank,
                           128) ||
           !make_tmap_bf16(&h->tm_sup, h->W_sup, (uint64_t)D.n_sum * D.d_seq, D.sum_rank, 64)))
        return fail(LLATTE_ERR_CUDA);
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(LLATTE_ERR_CUDA);
  *out = h;
  return LLATTE_OK;
}

}  // extern "C"

namespace {

// The export arguments, checked on the host.
int check_export(const llatte_handle* h, const llatte_attn_export* ex) {
  const llatte_dims& D = h->dims;
  if (ex->layer < 0 || ex->layer >= D.n_layers || ex->n_k < 1 || ex->n_k > 16 ||
      ex->n_hours < 0 || ex->n_hours > 8192 || !ex->recent || !ex->topk ||
      (ex->n_hours > 0) != (ex->event_age != nullptr) || (ex->n_hours > 0) != (ex->hours != nullptr))
    return LLATTE_ERR_ARG;
  if (D.n_q <= 0) return LLATTE_ERR_ARG;
  if (D.max_len > LLATTE_EXPORT_MAX_LEN) return LLATTE_ERR_UNSUPPORTED;
  return LLATTE_OK;
}

int forward_impl(llatte_handle* h, const void* values, const int64_t* offsets, int32_t B,
                 const void* context, const void* cand, const float* ages, float* out,
                 void* stream) {
  const llatte_dims& D = h->dims;
  if (B < 0 || B > D.max_batch) return LLATTE_ERR_ARG;
  if (B == 0) { h->last_B = 0; return LLATTE_OK; }
  if (!offsets) return LLATTE_ERR_ARG;  // values may be NULL when every history is empty
  if (D.d_ctx > 0 && !context) return LLATTE_ERR_ARG;
  if (D.n_q > 0 && !cand) return LLATTE_ERR_ARG;
  const bool has_out = D.d_out > 0 || D.n_q > 0;
  if (has_out && !out) return LLATTE_ERR_ARG;
  if (((uintptr_t)values | (uintptr_t)cand) & 15) return LLATTE_ERR_ARG;  // 16-byte rows
  if (D.n_sum > 0 && ((uintptr_t)out & 15)) return LLATTE_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const int L = D.n_layers, e = h->elem;
  const int d = D.d, r = D.rank, hr = D.heads * D.rank, f = D.ffn_mult * D.d;
  const PlanDev& p = h->plan;
  h->last_B = B;

  // Context term of every layer's query projection, one launch.  It depends
  // on nothing above, so outside profiling it runs on the side stream while
  // the plan and the gather run here; the first query projection waits for it.
  // With a low-rank query the term belongs to the down-projection (before
  // its RMSNorm): q_rank columns, fp16 for the tensor-core norm epilogue.
  // Per-head layers take the term of their non-absorbed W_q (h*d_h columns).
  bool ctx_join = false;
  const int rq = D.q_rank;
  const int hdh = D.heads * D.d_head;
  __half* ctx16 = (rq && h->use_tc) ? (__half*)h->ctxbias : nullptr;
  CtxWeights cw = {};
  int ctx_n = 0;
  {
    int64_t off = 0;
    for (int l = 0; l < L; ++l) {
      const bool ph = (h->heads_mask >> l) & 1u;
      cw.W[l] = rq ? h->layers[l].W_dqc : (ph ? h->layers[l].W_qhc : h->layers[l].W_qkc);
      cw.N[l] = rq ? rq : (ph ? hdh : hr);
      cw.off[l] = off;
      off += (int64_t)B * cw.N[l];
      ctx_n = std::max(ctx_n, cw.N[l]);
    }
  }
  if (D.d_ctx > 0) {
    if (h->profiling) {
      StepTimer t(h, s, ST_CTX);
      CK(launch_ctx_bias(e, context, cw, L, B, ctx_n, D.d_ctx, h->ctxbias, ctx16, s));
      t.done(1);
    } else {
      CK(cudaEventRecord(h->ev_fork, s));
      CK(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
      CK(launch_ctx_bias(e, context, cw, L, B, ctx_n, D.d_ctx, h->ctxbias, ctx16, h->side));
      CK(cudaEventRecord(h->ev_join, h->side));
      ctx_join = true;
    }
  }
  { StepTimer t(h, s, ST_PLAN); CK(launch_plan(h, offsets, B, s)); t.done(1); }
  { StepTimer t(h, s, ST_GATHER); CK(launch_gather(h, values, offsets, cand, ages, B, s)); t.done(1); }

  for (int l = 0; l < L; ++l) {
    const LayerDev& W = h->layers[l];
    void* Xh_l = h->Xh[l & 1];
    void* Xq_l = h->Xq[l & 1];
    void* Xh_n = h->Xh[(l + 1) & 1];
    void* Xq_n = h->Xq[(l + 1) & 1];
    const bool last = l == L - 1;
    const bool per_head = (h->heads_mask >> l) & 1u;   // MLA in its non-absorbed form

    const bool tc = h->use_tc != 0;
    // epilogue arguments shared by both paths
    NormArgs kv_norm = {};
    kv_norm.N = r; kv_norm.g = W.g_kv; kv_norm.eps = D.eps; kv_norm.M_dev = p.hist_total(l);
    kv_norm.M_max = h->max_rows_h; kv_norm.mode = NORM_PLAIN; kv_norm.dst = h->C;
    // Residual stream: bf16 storage keeps an fp16 copy of Z and of every
    // layer's query rows for the residual adds (the bf16 copies feed the
    // tensor cores); fp32 storage adds to the stored rows directly.
    const bool res16 = e == 2;
    NormArgs o_norm = {};
    o_norm.N = d; o_norm.g = W.g1; o_norm.eps = D.eps; o_norm.res_kind = RES_F16;
    // residual: the layer input rows (layer 0: the gathered inputs, exact in
    // the storage type)
    o_norm.resid = (l == 0 || !res16) ? Xq_l : h->Xqres[l & 1];
    o_norm.resid_kind = (l == 0 || !res16) ? RES_STORAGE : RES_F16;
    o_norm.M_dev = p.query_total(l); o_norm.M_max = h->max_rows_q; o_norm.mode = NORM_PLAIN;
    // on the tensor cores the FFN reads Z only as fp16 (its first operand and
    // its residual), so then the bf16 copy is not written
    const bool z16_only = tc && res16;
    // layers >= 1 (full-rank query, tensor cores): the query rows are read in
    // fp16, from the residual copy the previous layer's FFN wrote
    const bool q16 = tc && res16 && l >= 1 && !rq;
    o_norm.dst = z16_only ? nullptr : h->Z; o_norm.dst_res = res16 ? h->Zres : nullptr;
    NormArgs f_norm = {};
    f_norm.N = d; f_norm.resid = res16 ? h->Zres : h->Z;
    f_norm.resid_kind = res16 ? RES_F16 : RES_STORAGE; f_norm.res_kind = RES_F16;
    f_norm.g = W.g2; f_norm.eps = D.eps;
    f_norm.M_dev = p.query_total(l); f_norm.M_max = h->max_rows_q; f_norm.mode = NORM_SCATTER;
    f_norm.qoff_l = p.qoff(l); f_norm.n_l = p.nl(l); f_norm.hoff_n = p.hoff(l + 1);
    f_norm.qoff_n = p.qoff(l + 1); f_norm.n_n = p.nl(l + 1); f_norm.B = B; f_norm.n_q = D.n_q;
    // the next layer reads its query rows in fp16 on the tensor cores (full-rank
    // query), so then the bf16 copy is not written
    const bool next_q16 = tc && res16 && !rq && !last;
    f_norm.Xh_n = Xh_n; f_norm.Xq_n = next_q16 ? nullptr : Xq_n; f_norm.last = last;
    f_norm.Xq_res_n = (res16 && !last) ? h->Xqres[(l + 1) & 1] : nullptr;
    f_norm.out = out; f_norm.final_rows = D.d_out ? h->final_rows : nullptr;
    f_norm.zraw = (last && D.n_sum > 0) ? h->zraw : nullptr;
    f_norm.row_user = p.ruser(l);
    const LayerMaps& LM = h->lmaps[l];
    auto tcp = [&](const int64_t* Mdev, int64_t cap, int N, int K) {
      TcGemmParams q = {};
      q.M_dev = Mdev; q.M_cap = cap; q.N = N; q.K = K; q.status = p.status;
      return q;
    };

    {  // KV latent
      StepTimer t(h, s, ST_KV);
      if (tc) {
        TcGemmParams q = tcp(p.hist_total(l), h->max_rows_h, r, d);
        q.norm = kv_norm;
        q.D = (__nv_bfloat16*)h->C; q.ldd = r;
        CK(launch_tc_gemm(h->bn_kv, D.kv_norm ? TC_NORM : TC_STORE, h->tm_Xh[l & 1], LM.dkv, q,
                          h->num_sms, s, &h->tms_C));
        if (per_head) {
          // K | V = c_kv [W_uk ; W_uv]^T, every head's keys and values
          TcGemmParams k2 = tcp(p.hist_total(l), h->max_rows_h, 2 * hdh, r);
          k2.D = (__nv_bfloat16*)h->KV; k2.ldd = 2 * hdh;
          CK(launch_tc_gemm(pick_bn(2 * hdh), TC_STORE, h->tm_C, LM.ukv, k2, h->num_sms, s,
                            &h->tms_KV));
          t.done(2);
        } else {
          t.done(1);
        }
      } else {
        GemmArgs g = {};
        g.A = Xh_l; g.lda = d; g.W = W.W_dkv; g.M_dev = p.hist_total(l); g.M_max = h->max_rows_h;
        g.N = r; g.K = d;
        if (D.kv_norm) {
          g.D = h->acc32; g.ldd = r; g.epi = EPI_F32;
          CK(launch_gemm_simt(e, e, 4, g, s));
          kv_norm.acc = h->acc32;
          CK(launch_rownorm(e, kv_norm, s));
          t.done(2);
        } else {
          g.D = h->C; g.ldd = r; g.epi = EPI_STORE;
          CK(launch_gemm_simt(e, e, e, g, s));
          t.done(1);
        }
      }
    }
    {  // absorbed queries (+ per-user context term)
      if (ctx_join) {
        CK(cudaStreamWaitEvent(s, h->ev_join, 0));
        ctx_join = false;
      }
      StepTimer t(h, s, ST_Q);
      if (per_head) {
        // per-head query rows [rows, h*d_h] = R W_q,x^T + context term
        TcGemmParams q = tcp(p.query_total(l), h->max_rows_q, hdh, d);
        q.D = (__nv_bfloat16*)h->Qt; q.ldd = hdh;
        q.bias = h->ctxbias + cw.off[l]; q.seg_off = p.qoff(l); q.B = B;
        q.row_user = p.ruser(l);
        q.ab_f16 = q16 ? 1 : 0;
        CK(launch_tc_gemm(pick_bn(hdh), D.d_ctx > 0 ? TC_USERBIAS : TC_STORE,
                          q16 ? h->tm_Xqres[l & 1] : h->tm_Xq[l & 1], q16 ? LM.qh16 : LM.qh, q,
                          h->num_sms, s, &h->tms_Qh));
      } else if (rq) {
        // low-rank query: Cq = RMSNorm_{g_q}(R W_dq,x^T + context term of the
        // row's user), then the absorbed projection Qt = Cq (W_uk^T W_uq)^T
        NormArgs qn = {};
        qn.N = rq; qn.g = W.g_q; qn.eps = D.eps; qn.M_dev = p.query_total(l);
        qn.M_max = h->max_rows_q; qn.mode = NORM_PLAIN; qn.dst = h->Cq;
        if (tc) {
          if (D.d_ctx > 0) {
            qn.resid = ctx16 + cw.off[l]; qn.resid_kind = RES_F16;
            qn.resid_user = p.ruser(l);
          }
          TcGemmParams q1 = tcp(p.query_total(l), h->max_rows_q, rq, d);
          q1.norm = qn;
          CK(launch_tc_gemm(h->bn_dq, TC_NORM, h->tm_Xq[l & 1], LM.dq, q1, h->num_sms, s,
                            &h->tms_Cq));
          TcGemmParams q2 = tcp(p.query_total(l), h->max_rows_q, hr, rq);
          q2.D = (__nv_bfloat16*)h->Qt; q2.ldd = hr;
          CK(launch_tc_gemm(h->bn_q, TC_STORE, h->tm_Cq, LM.qk, q2, h->num_sms, s, &h->tms_Qt));
          t.done(2);
        } else {
          GemmArgs g = {};
          g.A = Xq_l; g.lda = d; g.W = W.W_dqx; g.D = h->acc32; g.ldd = rq;
          g.M_dev = p.query_total(l); g.M_max = h->max_rows_q; g.N = rq; g.K = d;
          g.epi = D.d_ctx > 0 ? EPI_USERBIAS_F32 : EPI_F32;
          g.bias = h->ctxbias + cw.off[l]; g.seg_off = p.qoff(l); g.B = B;
          CK(launch_gemm_simt(e, e, 4, g, s));
          qn.acc = h->acc32;
          CK(launch_rownorm(e, qn, s));
          GemmArgs g2 = {};
          g2.A = h->Cq; g2.lda = rq; g2.W = W.W_qk; g2.D = h->Qt; g2.ldd = hr;
          g2.M_dev = p.query_total(l); g2.M_max = h->max_rows_q; g2.N = hr; g2.K = rq;
          g2.epi = EPI_STORE;
          CK(launch_gemm_simt(e, e, e, g2, s));
          t.done(3);
        }
      } else if (tc) {
        TcGemmParams q = tcp(p.query_total(l), h->max_rows_q, hr, d);
        q.D = (__nv_bfloat16*)h->Qt; q.ldd = hr;
        q.bias = h->ctxbias + cw.off[l]; q.seg_off = p.qoff(l); q.B = B;
        q.row_user = p.ruser(l);
        q.ab_f16 = q16 ? 1 : 0;
        CK(launch_tc_gemm(h->bn_q, D.d_ctx > 0 ? TC_USERBIAS : TC_STORE,
                          q16 ? h->tm_Xqres[l & 1] : h->tm_Xq[l & 1], q16 ? LM.qk16 : LM.qk,
                          q, h->num_sms, s, &h->tms_Qt));
      } else {
        GemmArgs g = {};
        g.A = Xq_l; g.lda = d; g.W = W.W_qk; g.D = h->Qt; g.ldd = hr;
        g.M_dev = p.query_total(l); g.M_max = h->max_rows_q; g.N = hr; g.K = d;
        g.epi = D.d_ctx > 0 ? EPI_USERBIAS : EPI_STORE;
        g.bias = h->ctxbias + cw.off[l]; g.seg_off = p.qoff(l); g.B = B;
        CK(launch_gemm_simt(e, e, e, g, s));
      }
      if (!rq) t.done(1);
    }
    if (tc) {  // latent attention, tensor cores
      StepTimer t(h, s, ST_ATTN);
      AttnTcParams a = {};
      a.work = p.work + (int64_t)l * 2 * p.max_work; a.work_count = p.work_count + l;
      a.max_items = p.max_work; a.T = p.Tl(l); a.n = p.nl(l); a.hoff = p.hoff(l);
      a.qoff = p.qoff(l); a.n_q = D.n_q; a.heads = D.heads; a.Ot = (__nv_bfloat16*)h->Ot;
      a.status = p.status; a.inject_timeout = h->inject_timeout;
      if (per_head) CK(launch_attn_heads(h->tm_Qh, h->tm_KV, a, h->num_sms, s));
      else CK(launch_attn_tc(r, h->tm_Qt, h->tm_C, a, h->num_sms, s));
      t.done(1);
    } else {  // latent attention, CUDA cores
      StepTimer t(h, s, ST_ATTN);
      AttnArgs a = {};
      a.Qt = h->Qt; a.C = h->C; a.Ot = h->Ot; a.qoff = p.qoff(l); a.hoff = p.hoff(l);
      a.T = p.Tl(l); a.n = p.nl(l); a.Mq_dev = p.query_total(l); a.Mq_max = h->max_rows_q;
      a.B = B; a.heads = D.heads; a.r = r;
      CK(launch_attn_simt(e, a, s));
      t.done(1);
    }
    if (h->export_req && h->export_req->layer == l) {  // attention statistics of this layer
      const llatte_attn_export& ex = *h->export_req;
      ExportArgs x = {};
      x.Qt = h->Qt; x.C = per_head ? h->KV : h->C; x.qoff = p.qoff(l); x.hoff = p.hoff(l);
      x.evoff = offsets; x.T = p.Tl(l); x.n = p.nl(l); x.T0 = p.Tl(0);
      x.B = B; x.n_q = D.n_q; x.heads = D.heads; x.r = per_head ? 64 : r;
      if (per_head) { x.q_row = hdh; x.q_head = 64; x.c_row = 2 * hdh; x.c_head = 64; }
      else { x.q_row = (int64_t)D.heads * r; x.q_head = r; x.c_row = r; x.c_head = 0; }
      int n2 = 1;
      while (n2 < D.max_len) n2 <<= 1;
      x.n2 = n2; x.n_k = ex.n_k; x.n_hours = ex.n_hours; x.log2_scores = tc ? 1 : 0;
      x.event_age = ex.n_hours > 0 ? ex.event_age : nullptr;
      x.recent = ex.recent; x.topk = ex.topk; x.hours = ex.n_hours > 0 ? ex.hours : nullptr;
      StepTimer t(h, s, ST_EXPORT);
      CK(launch_attn_export(e, x, s));
      t.done(1);
    }
    {  // output projection + residual + RMSNorm
      StepTimer t(h, s, ST_O);
      if (tc) {
        TcGemmParams q = tcp(p.query_total(l), h->max_rows_q, d, per_head ? hdh : hr);
        q.norm = o_norm;
        const CUtensorMap& oa = per_head ? h->tm_Oh : h->tm_Ot;
        if (h->pair_norm)
          CK(launch_tc_gemm_pair(TC_NORM, oa, per_head ? LM.oh_pair : LM.ov_pair, q, h->num_sms, s));
        else
          CK(launch_tc_gemm(h->bn_o, TC_NORM, oa, per_head ? LM.oh : LM.ov, q, h->num_sms, s,
                            &h->tms_Zres));
        t.done(1);
      } else {
        GemmArgs g = {};
        g.A = h->Ot; g.lda = hr; g.W = W.W_ov; g.D = h->acc32; g.ldd = d;
        g.M_dev = p.query_total(l); g.M_max = h->max_rows_q; g.N = d; g.K = hr; g.epi = EPI_F32;
        CK(launch_gemm_simt(e, e, 4, g, s));
        o_norm.acc = h->acc32;
        CK(launch_rownorm(e, o_norm, s));
        t.done(2);
      }
    }
    if (tc && h->ffn_fused) {  // FFN up + SiLU + down + residual + RMSNorm, one kernel
      StepTimer t(h, s, ST_FFN);
      FfnTcParams q = {};
      q.M_dev = p.query_total(l); q.M_cap = h->max_rows_q; q.F = f; q.norm = f_norm;
      q.status = p.status;
      q.z_f16 = z16_only ? 1 : 0;
      CK(launch_ffn_pair(z16_only ? h->tm_Zres : h->tm_Z, z16_only ? LM.w1h_pair : LM.w1_pair,
                         LM.w2_pair, q, h->num_sms, s));
      t.done(1);
      continue;
    }
    {  // FFN up + SiLU
      StepTimer t(h, s, ST_FFN1);
      if (tc) {
        TcGemmParams q = tcp(p.query_total(l), h->max_rows_q, f, d);
        q.D = (__nv_bfloat16*)h->Hd; q.ldd = f;
        q.ab_f16 = z16_only ? 1 : 0;
        CK(launch_tc_gemm(h->bn_f1, TC_SILU, z16_only ? h->tm_Zres : h->tm_Z,
                          z16_only ? LM.w1h : LM.w1, q, h->num_sms, s, &h->tms_Hd));
      } else {
        GemmArgs g = {};
        g.A = h->Z; g.lda = d; g.W = W.W1; g.D = h->Hd; g.ldd = f;
        g.M_dev = p.query_total(l); g.M_max = h->max_rows_q; g.N = f; g.K = d; g.epi = EPI_SILU;
        CK(launch_gemm_simt(e, e, e, g, s));
      }
      t.done(1);
    }
    {  // FFN down + residual + RMSNorm, scattered into the next layer's rows
      StepTimer t(h, s, ST_FFN2);
      if (tc) {
        TcGemmParams q = tcp(p.query_total(l), h->max_rows_q, d, f);
        q.norm = f_norm;
        if (h->pair_norm) CK(launch_tc_gemm_pair(TC_NORM, h->tm_Hd, LM.w2_pair, q, h->num_sms, s));
        else CK(launch_tc_gemm(h->bn_f2, TC_NORM, h->tm_Hd, LM.w2, q, h->num_sms, s));
        t.done(1);
      } else {
        GemmArgs g = {};
        g.A = h->Hd; g.lda = f; g.W = W.W2; g.D = h->acc32; g.ldd = d;
        g.M_dev = p.query_total(l); g.M_max = h->max_rows_q; g.N = d; g.K = f; g.epi = EPI_F32;
        CK(launch_gemm_simt(e, e, 4, g, s));
        f_norm.acc = h->acc32;
        CK(launch_rownorm(e, f_norm, s));
        t.done(2);
      }
    }
  }
  if (D.d_out > 0) {
    StepTimer t(h, s, ST_READOUT);
    CK(launch_mean_rows(h->final_rows, p.qoff(L - 1), B, d, h->mean_rows,
                        h->readout_tc ? h->mean16 : nullptr, s));
    if (h->readout_tc) {
      // out = mean E^T on the tensor cores: the mean in bf16, fp32 out
      TcGemmParams q = {};
      q.M_host = B; q.M_dev = nullptr; q.M_cap = D.max_batch; q.N = D.d_out; q.K = d;
      q.status = p.status; q.Dp = out; q.slice_stride = 0; q.k_split = 1; q.groups = 1;
      q.ldp = D.d_out;
      CK(launch_tc_gemm(64, TC_F32, h->tm_mean16, h->tm_We, q, h->num_sms, s));
    } else {
      GemmArgs g = {};
      g.A = h->mean_rows; g.lda = d; g.W = h->W_e; g.D = out; g.ldd = D.d_out;
      g.M_host = B; g.M_dev = nullptr; g.M_max = B; g.N = D.d_out; g.K = d; g.epi = EPI_F32;
      CK(launch_gemm_simt(4, e, 4, g, s));
    }
    t.done(2);
  }
  if (D.n_sum > 0) {  // sequence summaries of the final query-token rows
    StepTimer t(h, s, ST_SUMMARY);
    const int N = D.n_sum * D.sum_rank, K = D.n_q * d;
    int S = 1;
    if (h->sum_tc) {
      S = summary_slices(B, N, h->sum_bn, K);
      TcGemmParams q = {};
      q.M_host = B; q.M_dev = nullptr; q.M_cap = B; q.N = N; q.K = K; q.status = p.status;
      q.Dp = h->sum_part; q.slice_stride = (int64_t)B * N; q.k_split = S;
      q.groups = 1; q.ldp = N;
      CK(launch_tc_gemm(h->sum_bn, TC_F32, h->tm_zraw, h->tm_sdown, q, h->num_sms, s));
    } else {
      GemmArgs g = {};
      g.A = h->zraw; g.lda = K; g.W = h->W_sdown; g.D = h->sum_part; g.ldd = N;
      g.M_host = B; g.M_dev = nullptr; g.M_max = B; g.N = N; g.K = K; g.epi = EPI_F32;
      CK(launch_gemm_simt(e, e, 4, g, s));
    }
    SummaryArgs sa = {};
    sa.P = h->sum_part; sa.S = S; sa.slice_stride = (int64_t)B * N;
    sa.H = h->sum_up_tc ? nullptr : h->sum_h;
    sa.H16 = (__nv_bfloat16*)h->sum_h16; sa.b_pad = h->sum_bpad;
    sa.B = B; sa.N = N;
    sa.rank = D.sum_rank; sa.d_seq = D.d_seq; sa.n_sum = D.n_sum; sa.Wt = h->W_sup; sa.out = out;
    CK(launch_summary_reduce(sa, s));
    if (h->sum_up_tc) {
      // out[b, k, :] = H16[k, b, :] W_up,k^T for every k, one batched GEMM
      TcGemmParams q = {};
      q.M_host = B; q.M_dev = nullptr; q.M_cap = B; q.N = D.d_seq; q.K = D.sum_rank;
      q.status = p.status; q.Dp = out; q.k_split = 1; q.groups = D.n_sum;
      q.a_group_rows = h->sum_bpad; q.w_group_rows = D.d_seq; q.d_group_off = D.d_seq;
      q.ldp = (int64_t)D.n_sum * D.d_seq;
      CK(launch_tc_gemm(64, TC_F32, h->tm_sh16, h->tm_sup, q, h->num_sms, s));
    } else {
      CK(launch_summary_up(e, sa, s));
    }
    t.done(3);
  }
  return LLATTE_OK;
}

}  // namespace

extern "C" {

int llatte_forward(llatte_handle* h, const void* values, const int64_t* offsets, int32_t B,
                   const void* context, const void* cand, float* out, void* stream) {
  if (!h || h->dims.d_time > 0) return LLATTE_ERR_ARG;     // the timestamp code needs ages
  return forward_impl(h, values, offsets, B, context, cand, nullptr, out, stream);
}

int llatte_forward_export(llatte_handle* h, const void* values, const int64_t* offsets, int32_t B,
                          const void* context, const void* cand, float* out,
                          const llatte_attn_export* ex, void* stream) {
  if (!h || !ex || h->dims.d_time > 0) return LLATTE_ERR_ARG;
  const int rc0 = check_export(h, ex);
  if (rc0 != LLATTE_OK) return rc0;
  h->export_req = ex;
  const int rc = forward_impl(h, values, offsets, B, context, cand, nullptr, out, stream);
  h->export_req = nullptr;
  return rc;
}

int llatte_forward_batch(llatte_handle* h, const llatte_batch* b, float* out,
                         const llatte_attn_export* ex, void* stream) {
  if (!h || !b) return LLATTE_ERR_ARG;
  if (h->dims.d_time > 0 && b->B > 0 && !b->event_age) return LLATTE_ERR_ARG;
  if (ex) {
    const int rc0 = check_export(h, ex);
    if (rc0 != LLATTE_OK) return rc0;
  }
  h->export_req = ex;
  const int rc = forward_impl(h, b->values, b->offsets, b->B, b->context, b->cand,
                              h->dims.d_time > 0 ? b->event_age : nullptr, out, stream);
  h->export_req = nullptr;
  return rc;
}

int llatte_plan_export(llatte_handle* h, int64_t* dst, void* stream) {
  if (!h || !dst) return LLATTE_ERR_ARG;
  const int B = h->last_B, L = h->dims.n_layers;
  cudaStream_t s = (cudaStream_t)stream;
  for (int l = 0; l < L; ++l) {
    CK(cudaMemcpyAsync(dst + (size_t)(2 * l) * (B + 1), h->plan.hist_off + l * h->plan.stride,
                       sizeof(int64_t) * (B + 1), cudaMemcpyDeviceToDevice, s));
    CK(cudaMemcpyAsync(dst + (size_t)(2 * l + 1) * (B + 1), h->plan.query_off + l * h->plan.stride,
                       sizeof(int64_t) * (B + 1), cudaMemcpyDeviceToDevice, s));
  }
  return LLATTE_OK;
}

int llatte_get_status(llatte_handle* h, int32_t* device_status) {
  if (!h || !device_status) return LLATTE_ERR_ARG;
  CK(cudaDeviceSynchronize());
  int32_t v = 0;
  CK(cudaMemcpy(&v, h->plan.status, sizeof(int32_t), cudaMemcpyDeviceToHost));
  CK(cudaMemset(h->plan.status, 0, sizeof(int32_t)));
  *device_status = v;
  return v ? LLATTE_ERR_DEVICE : LLATTE_OK;
}

int llatte_attn_form_mask(const llatte_handle* h, uint32_t* per_head_layers) {
  if (!h || !per_head_layers) return LLATTE_ERR_ARG;
  *per_head_layers = h->heads_mask;
  return LLATTE_OK;
}

int llatte_inject_timeout(llatte_handle* h, int enable) {
  if (!h || (enable != 0 && enable != 1)) return LLATTE_ERR_ARG;
  if (!h->use_tc || h->heads_mask == 0) return LLATTE_ERR_UNSUPPORTED;
  h->inject_timeout = enable;
  return LLATTE_OK;
}

int llatte_set_profiling(llatte_handle* h, int enable) {
  if (!h) return LLATTE_ERR_ARG;
  h->profiling = enable ? 1 : 0;
  return LLATTE_OK;
}

int llatte_profile_reset(llatte_handle* h) {
  if (!h) return LLATTE_ERR_ARG;
  int rc = drain_profile(h);
  for (int i = 0; i < ST_COUNT; ++i) { h->step_ms[i] = 0; h->step_launches[i] = 0; h->step_calls[i] = 0; }
  return rc;
}

int llatte_profile_step(llatte_handle* h, int step, const char** name, double* total_ms,
                        int64_t* kernel_launches, int64_t* calls) {
  if (!h || step < 0 || step >= ST_COUNT) return LLATTE_ERR_ARG;
  int rc = drain_profile(h);
  if (rc != LLATTE_OK) return rc;
  if (name) *name = kStepNames[step];
  if (total_ms) *total_ms = h->step_ms[step];
  if (kernel_launches) *kernel_launches = h->step_launches[step];
  if (calls) *calls = h->step_calls[step];
  return LLATTE_OK;
}

}  // extern "C"
