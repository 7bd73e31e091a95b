// Internal structures of the LLaTTE forward library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/llatte.h"

namespace llatte {

// Step kinds, for the optional per-step timing.
enum Step { ST_PLAN = 0, ST_GATHER, ST_CTX, ST_KV, ST_Q, ST_ATTN, ST_O, ST_FFN1, ST_FFN2,
            ST_READOUT, ST_FFN, ST_SUMMARY, ST_EXPORT, ST_COUNT };
extern const char* const kStepNames[ST_COUNT];

// Device-side pyramid plan.  Layer index l runs over 0..L where l = L is the
// virtual layer holding the final rows (its keep is unbounded).
struct PlanDev {
  int64_t* hist_off;   // [(L+1) * (max_batch+1)]  exclusive scan of T_{l,u}
  int64_t* query_off;  // [(L+1) * (max_batch+1)]  exclusive scan of n_{l,u} + n_q
  int32_t* T;          // [(L+1) * max_batch]
  int32_t* n;          // [(L+1) * max_batch]
  int64_t* totals;     // [(L+1) * 2]: sum T_l, sum (n_l + n_q)
  int32_t* status;     // device status word
  int32_t* work;       // attention work items, [(L) * max_work] (tensor-core path)
  int32_t* work_count; // [L]
  int32_t* work_next;  // [L] dynamic scheduling counters
  int32_t* item_off;   // [L][max_batch+1] scratch: first work item of each user
  int32_t* row_user;   // [L][max rows_q]: user of every query row of every layer
  int64_t row_user_stride;
  __host__ __device__ const int32_t* ruser(int l) const { return row_user + l * row_user_stride; }
  int64_t stride;      // max_batch + 1
  int32_t max_work;

  __host__ __device__ const int64_t* hoff(int l) const { return hist_off + l * stride; }
  __host__ __device__ const int64_t* qoff(int l) const { return query_off + l * stride; }
  __host__ __device__ const int32_t* Tl(int l) const { return T + l * (stride - 1); }
  __host__ __device__ const int32_t* nl(int l) const { return n + l * (stride - 1); }
  __host__ __device__ const int64_t* hist_total(int l) const { return totals + 2 * l; }
  __host__ __device__ const int64_t* query_total(int l) const { return totals + 2 * l + 1; }
};

struct LayerDev {
  void* W_dkv;     // [r, d]
  void* g_kv;      // [r]
  void* W_qk;      // [h*r, d]   absorbed W_uk^T W_q (x columns), scaled 1/sqrt(d_h)
                   //   low-rank query: [h*r, q_rank] absorbed W_uk^T W_uq
  float* W_qkc;    // [d_ctx, h*r] fp32 absorbed context columns, transposed (NULL if d_ctx == 0
                   //   or low-rank query)
  void* W_dqx;     // [q_rank, d] query down-projection, x columns (low-rank query)
  float* W_dqc;    // [d_ctx, q_rank] fp32 its context columns, transposed (NULL if d_ctx == 0)
  void* g_q;       // [q_rank] query-latent RMSNorm gain
  // per-head (non-absorbed) form of the layer, d_h = 64 (NULL otherwise)
  void* W_qh;      // [h*d_h, d] W_q's x columns, scaled log2(e)/sqrt(d_h)
  float* W_qhc;    // [d_ctx, h*d_h] fp32 its context columns (same scale), transposed
  void* W_ukv;     // [2*h*d_h, r] W_uk stacked on W_uv
  void* W_oh;      // [d, h*d_h] W_o
  void* W_ov;      // [d, h*r]   absorbed W_o W_uv
  void* g1;        // [d]
  void* W1;        // [f, d]
  void* W1h;       // [f, d] fp16 copy of W1 (the FFN's first product takes fp16 Z)
  void* W_q16;     // fp16 copy of the layer's query weight (W_qk, or W_qh in the per-head
                   //   form) for layers >= 1: their query rows are read in fp16
  void* W2;        // [d, f]
  void* g2;        // [d]
};

struct ProfRec { int step; cudaEvent_t a, b; int launches; };

// TMA descriptors of one layer's weights (B operands of the tensor-core GEMMs).
struct LayerMaps {
  CUtensorMap dkv, qk, ov, w1, w2, w1_pair, w2_pair, ov_pair, dq;
  CUtensorMap w1h_pair;                 // fp16 W1, 64-row boxes (fused FFN)
  CUtensorMap w1h;                      // fp16 W1, bn_f1-row boxes (FFN-up GEMM)
  CUtensorMap qk16, qh16;               // fp16 query weights (layers >= 1, full-rank query)
  CUtensorMap qh, ukv, oh, oh_pair;     // per-head form
};

}  // namespace llatte

struct llatte_handle {
  llatte_dims dims;
  int device;
  int elem;                       // bytes per stored element
  int use_tc;                     // tensor-core (tcgen05) path for bf16
  int num_sms;
  llatte::LayerDev layers[LLATTE_MAX_LAYERS];
  void* W_e;                      // [d_out, d]
  // sequence summaries: the stacked bottleneck projections, the output
  // projections transposed, the final query-token rows and the split-K partials
  void* W_sdown;                  // [n_sum * sum_rank, n_q * d]
  void* W_sup;                    // [n_sum * d_seq, sum_rank] (sum_up_tc), else
                                  // transposed: [n_sum][sum_rank][d_seq]
  void* zraw;                     // [max_batch, n_q * d] storage type
  float* sum_part;                // [k slices][rows][n_sum * sum_rank] fp32
  float* sum_h;                   // [max_batch, n_sum * sum_rank] fp32
  void* sum_h16;                  // [n_sum][sum_bpad][sum_rank] bf16 (sum_up_tc)
  int64_t sum_bpad;               // max_batch rounded up to 128
  int sum_tc;                     // bottleneck GEMM on the tensor cores
  int sum_bn;                     // its tile width
  int sum_up_tc;                  // output projections as one batched tensor-core GEMM
  std::vector<void*> allocs;

  // workspace
  llatte::PlanDev plan;
  int64_t max_rows_h, max_rows_q;
  void* Xh[2];
  void* Xq[2];
  void* C;
  void* Qt;
  void* Ot;
  void* Z;
  void* Hd;
  void* Cq;            // [max_rows_q, q_rank] normalised query latent (low-rank query)
  void* Zres;          // fp16 residual copy of Z (bf16 storage only; NULL for fp32)
  void* Xqres[2];      // fp16 residual copy of the query rows (bf16 storage only)
  float* acc32;        // fp32 pre-norm rows (CUDA-core path)
  float* ctxbias;      // [n_layers][B][h*r] (this forward's B)
  float* final_rows;   // [max_rows_q, d] fp32 (readout only)
  float* mean_rows;    // [max_batch, d] fp32
  void* mean16;        // [max_batch, d] bf16 copy: the tensor-core readout's operand
  size_t ws_bytes;
  int last_B;

  // tensor-core path: TMA descriptors of the A operands and the weights,
  // and the tile width (BN) of each GEMM
  CUtensorMap tm_Xh[2], tm_Xq[2], tm_Ot, tm_Z, tm_Hd, tm_Cq;
  CUtensorMap tm_Zres;            // fp16 Z (the fused FFN's first operand and its residual)
  CUtensorMap tm_Xqres[2];        // fp16 query rows (the query projection's operand, layers >= 1)
  llatte::LayerMaps lmaps[LLATTE_MAX_LAYERS];
  int bn_kv, bn_q, bn_o, bn_f1, bn_f2, bn_dq;
  int attn_keys;                  // keys per attention tile (tensor-core path)
  int ffn_fused;                  // FFN up + SiLU + down in one kernel (d = 256)
  int pair_norm;                  // output / FFN-down projections on SM pairs (d = 512)
  CUtensorMap tm_Qt, tm_C;        // attention operands: [sum q * h, r] and [sum T, r]
  // store maps of the GEMM outputs (boxes of 32 rows x 32 columns): latent C,
  // the per-head K | V rows, the query rows ([rows, h r] and per-head
  // [rows, h d_h]), the low-rank query latent, fp16 Z, the FFN hidden rows
  CUtensorMap tms_C, tms_KV, tms_Qt, tms_Qh, tms_Cq, tms_Zres, tms_Hd;
  CUtensorMap tm_zraw, tm_sdown;  // summary bottleneck GEMM operands
  // per-head attention form: bit l = layer l runs it; its K | V rows, and the
  // query / output rows laid out [rows, h*d_h] (in the Qt / Ot memory)
  uint32_t heads_mask;
  int inject_timeout;             // failure-detection test: the next forwards' per-head
                                  //   attention runs a wait out on purpose
  void* KV;                       // [max_rows_h, 2*h*d_h]
  CUtensorMap tm_Qh, tm_KV, tm_Oh;
  CUtensorMap tm_sh16, tm_sup;    // summary output-projection GEMM operands
  CUtensorMap tm_mean16, tm_We;   // readout GEMM operands (readout_tc)
  int readout_tc;                 // the readout projection runs on the tensor cores

  // attention-probability export requested for the forward in progress
  const llatte_attn_export* export_req;

  // the per-user context term runs on a side stream, beside the plan and
  // the gather (forked from and joined back into the caller's stream)
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;

  // profiling
  int profiling;
  std::vector<llatte::ProfRec> pending;
  std::vector<cudaEvent_t> event_pool;
  double step_ms[llatte::ST_COUNT];
  int64_t step_launches[llatte::ST_COUNT];
  int64_t step_calls[llatte::ST_COUNT];
};

namespace llatte {

// ---- launchers (each returns cudaGetLastError()) ----
cudaError_t launch_plan(const llatte_handle* h, const int64_t* offsets, int B, cudaStream_t s);
// The plan kernel on caller-described storage (no work lists).
cudaError_t launch_plan_on(const PlanDev& p, const llatte_dims& d, int64_t max_total,
                           const int64_t* offsets, int B, cudaStream_t s);
// Layer-0 rows from the inputs; with ages != NULL (d_time > 0) the rows taken
// from `values` get the timestamp code on their first d_time dims.
cudaError_t launch_gather(const llatte_handle* h, const void* values, const int64_t* offsets,
                          const void* cand, const float* ages, int B, cudaStream_t s);

// CUDA-core path
struct GemmArgs {
  const void* A; int64_t lda;        // [M, K]
  const void* W;                     // [N, K] row-major
  void* D; int64_t ldd;              // [M, N]
  int64_t M_host; const int64_t* M_dev;  // M from device when M_dev != NULL
  int64_t M_max;                     // grid bound
  int N, K;
  int epi;                           // EPI_*
  const float* bias; const int64_t* seg_off; int B;  // EPI_USERBIAS
};
enum { EPI_STORE = 0, EPI_USERBIAS, EPI_SILU, EPI_F32, EPI_USERBIAS_F32 };
cudaError_t launch_gemm_simt(int elem_a, int elem_w, int elem_d, const GemmArgs& g, cudaStream_t s);

// Element type of a residual-stream buffer.
enum { RES_STORAGE = 0, RES_F32 = 1, RES_F16 = 2 };

struct NormArgs {
  const float* acc; int N;           // [M, N] fp32 rows
  const void* resid;                 // [M, N] residual or NULL
  int resid_kind;                    // RES_STORAGE / RES_F32 / RES_F16
  const int32_t* resid_user;         // non-NULL: the residual is per user, [B, N], row
                                     //   resid_user[m] for row m (RES_F16 only)
  const void* g; float eps;
  const int64_t* M_dev; int64_t M_max;
  int mode;                          // NORM_PLAIN / NORM_SCATTER
  int res_kind;                      // type of the residual copies written below
  void* dst; void* dst_res;          // NORM_PLAIN: [M, N] storage type (+ optional residual copy)
  // NORM_SCATTER (FFN2 output of layer l -> inputs of layer l+1 / outputs)
  const int64_t *qoff_l, *hoff_n, *qoff_n; const int32_t *n_l, *n_n; int B; int n_q;
  void* Xh_n; void* Xq_n; void* Xq_res_n; int last; float* out; float* final_rows;
  // last layer with sequence summaries: the query-token rows go, in the
  // storage type, to zraw[u * n_q + j] instead of the fp32 output
  void* zraw;
  const int32_t* row_user;           // user of each query row of layer l (tensor-core path)
};
// NORM_NONE (fused FFN kernel only): the block's output rows as they are, no
// residual and no norm, stored in the storage type to dst (the action
// tokenizer's MLP_act).
enum { NORM_PLAIN = 0, NORM_SCATTER = 1, NORM_NONE = 2 };
cudaError_t launch_rownorm(int elem, const NormArgs& a, cudaStream_t s);

struct AttnArgs {
  const void* Qt;                    // [sum q, h*r]
  const void* C;                     // [sum T, r]
  void* Ot;                          // [sum q, h*r]
  const int64_t *qoff, *hoff; const int32_t *T, *n;
  const int64_t* Mq_dev; int64_t Mq_max;
  int B, heads, r;
};
cudaError_t launch_attn_simt(int elem, const AttnArgs& a, cudaStream_t s);

// Per-user context term of every layer's absorbed query projection.
// Per layer l: W[l] [d_ctx, N[l]] fp32; the term of user u, column n goes to
// element off[l] + u * N[l] + n of the output.
struct CtxWeights {
  const float* W[LLATTE_MAX_LAYERS];
  int N[LLATTE_MAX_LAYERS];
  int64_t off[LLATTE_MAX_LAYERS];
};
// out (fp32), or out16 (fp16) when out16 != NULL, laid out as CtxWeights says;
// N_max = the largest N[l].
cudaError_t launch_ctx_bias(int elem, const void* ctx, const CtxWeights& w, int L, int B,
                            int N_max, int dc, float* out, __half* out16, cudaStream_t s);
// Split scale * (a [rows, d + dc] matrix) into its first d columns (storage
// type, [rows, d]) and its last dc columns (fp32, transposed: [dc, rows]).
cudaError_t launch_split_ctx_cols(int elem, const void* src, int rows, int d, int dc, void* dst_x,
                                  float* dst_c, float scale, cudaStream_t s);

// Sequence summaries after the bottleneck GEMM: H = SiLU(sum of the S split-K
// partial rows) (reduce), then out[b, k, :] = H[b, k-block] W_up,k^T (up, on
// CUDA cores; the tensor-core path runs it as a batched GEMM instead).
struct SummaryArgs {
  const float* P; int S; int64_t slice_stride;   // P[s * slice_stride + b * N + j]
  float* H;                                      // [B, N] fp32, or NULL and:
  __nv_bfloat16* H16; int64_t b_pad;             // [n_sum][b_pad][rank] bf16
  int B, N, rank, d_seq, n_sum;                  // N = n_sum * rank
  const void* Wt;                                // [n_sum][rank][d_seq] storage type
  float* out;                                    // [B, n_sum, d_seq]
};
cudaError_t launch_summary_reduce(const SummaryArgs& a, cudaStream_t s);
cudaError_t launch_summary_up(int elem, const SummaryArgs& a, cudaStream_t s);
// fp16 copy of n bf16 values.
cudaError_t launch_bf16_to_f16(const void* src, void* dst, int64_t n, cudaStream_t s);
// dst[c, r] = src[r, c] for a [rows, cols] matrix of the storage type.
cudaError_t launch_transpose(int elem, const void* src, int64_t rows, int64_t cols, void* dst,
                             cudaStream_t s);

// Attention-probability statistics of one layer's query tokens (see the
// attention-export call of the public header).
struct ExportArgs {
  const void* Qt; const void* C;                 // the layer's absorbed queries and latent keys
  const int64_t *qoff, *hoff, *evoff;            // layer query / history offsets, input offsets
  const int32_t *T, *n, *T0;                     // layer keys, kept history rows, input lengths
  int B, n_q, heads, r, n2, n_k, n_hours, log2_scores;
  // element strides: query (row m, head j) at Qt + m q_row + j q_head; key
  // row t of head j at C + t c_row + j c_head (absorbed: h r, r, r, 0;
  // per-head form: h 64, 64, 2 h 64, 64 with C = the K | V rows)
  int64_t q_row, q_head, c_row, c_head;
  const float* event_age;                        // [sum T0] hours, or NULL
  float *recent, *topk, *hours;                  // [B, n_q, h, n_k] x2, [B, n_q, h, n_hours]
};
size_t attn_export_smem(int n2, int r, int n_hours);
cudaError_t launch_attn_export(int elem, const ExportArgs& a, cudaStream_t s);

cudaError_t launch_mean_rows(const float* rows, const int64_t* qoff, int B, int d, float* mean,
                             void* mean16,
                             cudaStream_t s);
// W_q has dq + d_ctx columns (dq = d, or q_rank for W_uq of a low-rank query).
cudaError_t launch_absorb(int elem, const void* W_q, const void* W_uk, const void* W_uv,
                          const void* W_o, int d, int dq, int d_ctx, int heads, int d_head, int r,
                          float qscale, void* W_qk, float* W_qkc, void* W_ov, cudaStream_t s);

}  // namespace llatte
