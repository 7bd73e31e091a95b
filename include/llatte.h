/*
 * llatte.h - C ABI of the B200 (sm_100a) LLaTTE sequence-module forward pass.
 *
 * What it computes (LLaTTE notes, huaxiaozhuan.com, appendix A.2 "Sequence
 * Module" and A.3 "Multi-head Latent Attention"; target-aware query from the
 * daiwk.github.io notes, "core formula"):
 *
 *   per user u: history tokens x_1..x_T (earliest first), n_q query tokens
 *   (candidates), a context vector c.  Fused input = [history ; query tokens].
 *   For each layer l with keep_l:
 *     n      = min(T, keep_l)                  kept history rows
 *     R      = [last n history rows ; query tokens]        (query rows)
 *     c_kv   = RMSNorm_{g_kv}(H W_dkv^T)       latent K = V, rank r, all T rows
 *     per head j:  q~ = (W_uk,j^T W_q,j) [R_i ; c] / sqrt(d_h)
 *                  a  = softmax over visible keys t of q~ . c_kv,t
 *                  o~ = sum_t a_t c_kv,t
 *     A      = sum_j (W_o,j W_uv,j) o~_j
 *     Z      = RMSNorm_{g1}(R + A)
 *     X      = RMSNorm_{g2}(Z + W2 SiLU(W1 Z))
 *     history <- X[:n], query tokens <- X[n:], T <- n
 *   With q_rank > 0 the query is low-rank and normalised (appendix A.3, first
 *   display): q~ = (W_uk,j^T W_up,j^Q) RMSNorm_{g_q}(W_down^Q [R_i ; c]) / sqrt(d_h),
 *   the down-projection taking the target-aware input [x ; c].
 *   With d_time > 0 every history token first gets an additive timestamp code
 *   on its first d_time dims (appendix A.2 item 1; the pages give no formula:
 *   the Transformer's sinusoidal code of the event's age a in hours before
 *   the request is the reading taken): dims 2i, 2i+1 add sin(a w_i), cos(a w_i),
 *   w_i = 10000^(-2i/d_time).  Query tokens carry no timestamp.
 *   Visibility: a history query at position p sees keys t <= p; a query token
 *   sees every current history key and no query token; no key -> zero output.
 *   Output: the final query-token rows; or, with d_out > 0, W_e times the mean
 *   of the final layer's rows; or, with n_sum > 0, the sequence summaries
 *   Z_seq^(k) = W_up,k SiLU(W_down,k Flatten(Z_raw)), k = 1..n_sum, of the
 *   final query-token rows Z_raw [n_q, d] flattened row-major (token 0 first)
 *   (appendix A.2 item 4 "Sequence Summaries"; the pages call each map a
 *   low-rank adapted MLP and give no formula: a SiLU MLP whose hidden layer
 *   is the rank sum_rank bottleneck, without biases, is the reading taken).
 *
 * Conventions
 *   - All matrices are row-major [out, in] as on the pages.
 *   - dtype LLATTE_BF16: activations/weights in bfloat16, fp32 accumulation,
 *     fp32 softmax and RMSNorm statistics.  LLATTE_FP32: everything fp32 on
 *     CUDA cores (no tensor-core tf32).
 *   - Every call returns LLATTE_OK (0) or a negative LLATTE_ERR_* code; bad
 *     arguments are rejected on the host before anything is launched.
 *   - Faults that only the device can see (offsets not monotone, a user
 *     longer than max_len, a batch larger than max_total, a bounded wait that
 *     ran out) set bits in a device status word instead of trapping; the
 *     forward then does no further work and `out` is unspecified.
 *     llatte_get_status reads and clears that word.
 */
#ifndef LLATTE_H
#define LLATTE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LLATTE_MAX_LAYERS 16

enum {
  LLATTE_OK = 0,
  LLATTE_ERR_ARG = -1,          /* null pointer, bad size or bad schedule      */
  LLATTE_ERR_UNSUPPORTED = -2,  /* dims outside what the kernels implement     */
  LLATTE_ERR_CUDA = -3,         /* a CUDA runtime call failed                  */
  LLATTE_ERR_OOM = -4,          /* device allocation failed                    */
  LLATTE_ERR_DEVICE = -5        /* device status word is non-zero              */
};

enum { LLATTE_BF16 = 0, LLATTE_FP32 = 1 };

/* Bits of the device status word. */
enum {
  LLATTE_DEV_BAD_OFFSETS = 1,   /* offsets decrease or are negative            */
  LLATTE_DEV_TOO_LONG = 2,      /* a history longer than max_len               */
  LLATTE_DEV_TOO_MANY_ROWS = 4, /* sum of lengths above max_total              */
  LLATTE_DEV_TIMEOUT = 8,       /* a bounded device wait gave up               */
  LLATTE_DEV_BAD_ID = 16        /* tokenizer: an id outside its embedding table */
};

/*
 * Model dimensions (sizes and pyramid schedule).
 *   d, heads, d_head      token width, heads h, head width d_h (scale 1/sqrt(d_h))
 *   rank                  MLA latent rank r
 *   d_ctx                 context width (0 = no context)
 *   n_q                   query tokens per user (0 allowed)
 *   n_layers, keep[]      layers and, per layer, the number of most recent
 *                         HISTORY rows kept (non-increasing; 0 = cross mode)
 *   d_out                 readout width (0 = output the final query-token rows)
 *   ffn_mult              FFN hidden = ffn_mult * d
 *   dtype                 LLATTE_BF16 or LLATTE_FP32
 *   kv_norm               1 = RMSNorm on the KV latent (the pages' form), 0 = none
 *   eps                   RMSNorm epsilon
 *   max_batch             largest B a forward may pass
 *   max_len               longest history a user may have
 *   max_total             largest sum of lengths in one batch (0 = max_batch*max_len)
 *   n_sum                 sequence summaries (0 = none; needs n_q > 0 and d_out == 0;
 *                         at most LLATTE_MAX_SUMMARIES)
 *   sum_rank, d_seq       bottleneck width (1 .. 1024) and width (even) of each summary
 *   q_rank                rank of the low-rank RMSNorm'd query (0 = full-rank W_q;
 *                         at most 1024)
 *   d_time                dims carrying the timestamp code (even, <= d; 0 = none)
 *   attn_form             which form of MLA each layer runs (the same function):
 *                         LLATTE_ATTN_AUTO (per layer, the cheaper one),
 *                         LLATTE_ATTN_ABSORBED (latent-space multi-query attention)
 *                         or LLATTE_ATTN_PER_HEAD (K, V = split(c_kv W_up^KV), scores
 *                         over d_h; needs bf16, d_h = 64, q_rank = 0 and the
 *                         tensor-core dims, else LLATTE_ERR_UNSUPPORTED)
 */
typedef struct {
  int32_t d, heads, d_head, rank, d_ctx, n_q, n_layers;
  int32_t keep[LLATTE_MAX_LAYERS];
  int32_t d_out, ffn_mult, dtype, kv_norm;
  float eps;
  int32_t max_batch;
  int64_t max_len;
  int64_t max_total;
  int32_t n_sum, sum_rank, d_seq;
  int32_t q_rank;
  int32_t d_time;
  int32_t attn_form;
} llatte_dims;

enum { LLATTE_ATTN_AUTO = 0, LLATTE_ATTN_ABSORBED = 1, LLATTE_ATTN_PER_HEAD = 2 };

#define LLATTE_MAX_SUMMARIES 16

/*
 * Weights of one layer, non-absorbed, in `dtype` (row-major [out, in]):
 *   W_dkv [r, d]        KV down-projection         g_kv [r]   latent RMSNorm gain
 *   W_q   [h*d_h, d+d_ctx]  query projection of [x ; c]
 *   W_uk  [h*d_h, r]    K up-projection            W_uv [h*d_h, r] V up-projection
 *   W_o   [d, h*d_h]    output projection          g1 [d]     post-attention gain
 *   W1    [ffn_mult*d, d]   W2 [d, ffn_mult*d]     g2 [d]     post-FFN gain
 * With q_rank > 0, W_q is not read (may be NULL) and the query comes from
 *   W_dq  [q_rank, d+d_ctx] query down-projection  g_q [q_rank] its RMSNorm gain
 *   W_uq  [h*d_h, q_rank]   query up-projection
 * (all three ignored, and may be NULL, when q_rank == 0).
 */
typedef struct {
  const void *W_dkv, *g_kv, *W_q, *W_uk, *W_uv, *W_o, *g1, *W1, *W2, *g2;
  const void *W_dq, *g_q, *W_uq;
} llatte_layer_w;

/*
 * Weights of one sequence summary k, in `dtype` (row-major [out, in]):
 *   W_down [sum_rank, n_q*d]   bottleneck projection of the flattened rows
 *   W_up   [d_seq, sum_rank]   output projection
 */
typedef struct {
  const void *W_down, *W_up;
} llatte_summary_w;

typedef struct llatte_handle llatte_handle;

/*
 * Create a handle on the current CUDA device.  The weights (host memory if
 * weights_on_device == 0, device memory otherwise) are copied; the caller may
 * free them afterwards.  The absorbed matrices W_uk^T W_q / sqrt(d_h) and
 * W_o W_uv are formed on the device in fp32 and stored in `dtype`.  W_e is
 * [d_out, d] (ignored when d_out == 0); summaries points to n_sum
 * llatte_summary_w (ignored, and may be NULL, when n_sum == 0).  The handle
 * owns a workspace sized from max_batch / max_total; llatte_workspace_bytes
 * reports its size.  Synchronous.
 */
int llatte_create(llatte_handle** handle, const llatte_dims* dims,
                  const llatte_layer_w* layers, const void* W_e,
                  const llatte_summary_w* summaries, int weights_on_device);

/*
 * One batch of inputs, for llatte_forward_batch (the fields of llatte_forward
 * plus the event ages):
 *   event_age  device float [offsets[B]]: hours before the request of every
 *              history event, same jagged layout as values; required when
 *              d_time > 0 (otherwise ignored, may be NULL); the code keeps
 *              fp32 accuracy for ages below 4e5 hours
 */
typedef struct {
  const void* values;
  const int64_t* offsets;
  int32_t B;
  const void* context;
  const void* cand;
  const float* event_age;
} llatte_batch;

/*
 * One forward pass, asynchronous on `stream` (a cudaStream_t; NULL = legacy
 * default stream), with no host synchronisation.
 *   values  device [offsets[B] rows, d] in dtype: all users' histories, user u
 *           in rows offsets[u] .. offsets[u+1]-1, earliest event first;
 *           16-byte aligned (as are cand and context); may be NULL when
 *           every history is empty
 *   offsets device int64 [B+1], non-decreasing, offsets[0] >= 0
 *   B       number of users, 0 <= B <= max_batch (B = 0 launches nothing)
 *   context device [B, d_ctx] in dtype (may be NULL when d_ctx == 0)
 *   cand    device [B, n_q, d] in dtype (may be NULL when n_q == 0)
 *   out     device fp32 [B, n_q, d] (d_out == 0, n_sum == 0), [B, d_out]
 *           (d_out > 0) or [B, n_sum, d_seq] (n_sum > 0, 16-byte aligned)
 * Inputs are only read; `out` is the only caller memory written.  Calls on
 * one handle must not overlap in time (they share its workspace).  With
 * d_time > 0 it returns LLATTE_ERR_ARG (the ages are needed: use
 * llatte_forward_batch).
 */
int llatte_forward(llatte_handle* handle, const void* values, const int64_t* offsets,
                   int32_t B, const void* context, const void* cand, float* out,
                   void* stream);

/*
 * Copy the pyramid plan of the most recent forward (for bit-exact checks):
 * for every layer l = 0..n_layers-1 the history-row offsets then the
 * query-row offsets, dst = device int64 [n_layers][2][B+1] with B the last
 * forward's batch.  History rows of layer l: T_{l,u} = hist[u+1]-hist[u];
 * query rows: n_{l,u} + n_q = query[u+1]-query[u].  Asynchronous on stream.
 */
int llatte_plan_export(llatte_handle* handle, int64_t* dst, void* stream);

/*
 * Synchronise the device, read the status word into *device_status (0 = no
 * fault) and clear it.  Returns LLATTE_ERR_DEVICE when it was non-zero.
 */
int llatte_get_status(llatte_handle* handle, int32_t* device_status);

/*
 * The form of MLA each layer runs on this handle (bit l set: the per-head
 * form, K, V = split(c_kv W_up^KV) with scores over d_h; clear: the absorbed
 * latent-space form).  For cost accounting; the result does not depend on it.
 */
int llatte_attn_form_mask(const llatte_handle* handle, uint32_t* per_head_layers);

/*
 * Failure-detection aid; the paper has no counterpart.  Every wait inside the
 * tensor-core kernels is bounded: a wait that exceeds its limit records
 * LLATTE_DEV_TIMEOUT in the status word, and the kernel winds down (it lets
 * its own loads and matrix products in flight finish first) instead of
 * hanging.  With enable = 1 the forward calls that follow on this handle make
 * such a wait run out on purpose: in the attention of every layer in MLA's
 * per-head form, each CTA's matrix-product issuer, once its first products
 * and tiles are in flight, waits 20 us for an event that never happens.
 * enable = 0 switches that off.
 *
 * A forward during which a wait ran out leaves `out` unspecified and the
 * status bit set; the handle stays usable, and the next forward without the
 * injection computes the usual result.  Returns LLATTE_ERR_UNSUPPORTED when no
 * layer of the handle runs in the per-head form on the tensor cores (see
 * llatte_attn_form_mask), LLATTE_ERR_ARG for another enable value.
 */
int llatte_inject_timeout(llatte_handle* handle, int enable);

/* Bytes of device workspace a handle with these dims allocates (0 on bad dims). */
size_t llatte_workspace_bytes(const llatte_dims* dims);

/* Human-readable name of an LLATTE_* return code. */
const char* llatte_error_string(int code);

/*
 * Per-step device timing, a profiling aid.  With profiling enabled every
 * forward records a CUDA event pair on its stream around each step (plan,
 * gather, ctx_bias, kv, q, attn, o, ffn1, ffn2, readout, ffn when the FFN
 * runs as one fused kernel, summary, and attn_export); llatte_profile_step
 * synchronises on the recorded events and returns, for step index `step`
 * (0 .. 12), its name, the
 * accumulated milliseconds, the number of kernels the
 * step launched and the number of times it ran since the last reset.
 * Returns LLATTE_ERR_ARG for a step index out of range.
 */
int llatte_set_profiling(llatte_handle* handle, int enable);
int llatte_profile_reset(llatte_handle* handle);
int llatte_profile_step(llatte_handle* handle, int step, const char** name, double* total_ms,
                        int64_t* kernel_launches, int64_t* calls);

/*
 * The pyramid plan of one batch computed without allocating any device
 * memory, for callers that cannot call cudaMalloc where they need it (code
 * running under another framework's memory pool or allocator hook, or with
 * all device memory reserved up front).  It needs no handle.  The paper has
 * no counterpart of this call: it only serves such callers.
 *
 *   dims       host; uses n_layers, keep[], n_q, max_batch, max_len, max_total
 *   offsets    device int64 [B+1], as for llatte_forward
 *   B          0 <= B <= min(dims->max_batch, LLATTE_PLAN_STATIC_MAX_BATCH)
 *   plan_out   device int64 [n_layers][2][B+1]: the same values and layout as
 *              llatte_plan_export after llatte_forward on this batch
 *   status_out device int32: 0, or the LLATTE_DEV_* bits of a rejected batch
 *              (then plan_out holds zeros)
 *
 * Its scratch is one fixed device array of about 1.7 MB inside the library,
 * held on every GPU that loads the library until the process exits.  A batch
 * larger than LLATTE_PLAN_STATIC_MAX_BATCH users returns
 * LLATTE_ERR_UNSUPPORTED without launching anything.  The first call on a
 * device looks up that array's device address (with the device current);
 * make the first call before any stream capture.  That address is kept for
 * the life of the process: do not call this across a reset of the device or
 * of its primary context (the array then moves).  Every call on a device
 * shares the array: calls that can run at the same time on the GPU race, so
 * order them (one stream, or synchronise in between).  Asynchronous on
 * `stream`; it calls no cudaMalloc or cudaFree.
 */
#define LLATTE_PLAN_STATIC_MAX_BATCH 4096
int llatte_plan_static(const llatte_dims* dims, const int64_t* offsets, int32_t B,
                       int64_t* plan_out, int32_t* status_out, void* stream);

/*
 * Self-check of an arithmetic building block; the paper has no counterpart.
 * The absorbed-form attention softmax computes one probability pair in eight
 * with an
 * exponential built from fused multiply-adds (range reduction x = j + f,
 * |f| <= 1/2, a fitted cubic for 2^f, j added to the exponent field) instead
 * of the special-function unit.  This evaluates exactly that device function:
 *
 *   x     device float [n], inputs (<= 64; x <= -125, -inf and NaN give 0)
 *   y     device float [n], y[i] ~ 2^x[i], relative error below 1e-4
 *   y_hw  device float [n] or NULL: 2^x[i] from the hardware ex2.approx
 *
 * Returns LLATTE_ERR_ARG for n < 0 or a NULL x / y with n > 0.  Asynchronous
 * on `stream`; allocates nothing.
 */
int llatte_exp2_eval(const float* x, float* y, float* y_hw, int64_t n, void* stream);

/*
 * Attention-probability statistics (appendix A.4 "Attention Weight
 * Distribution": how much attention the query tokens give to the most recent
 * events, to the events with the largest weights, and by hours before the
 * request).  For layer `layer`, every (user u, query token i, head j) row of
 * P = softmax over that layer's history keys gives, for k = 2^0 .. 2^(n_k-1):
 *   recent [B, n_q, h, n_k]  sum of P over the k most recent keys
 *   topk   [B, n_q, h, n_k]  sum of the k largest entries of P
 * and, with n_hours > 0 and the age of every input event in hours before the
 * request (event_age, device float, same jagged layout as values):
 *   hours  [B, n_q, h, n_hours]  sum of P over keys with floor(age) = b, the
 *                                last bin also taking every older key
 * (a user without keys gives zeros).  The keys of layer l are the user's
 * most recent T_l events.  Reading: the pages plot these curves aggregated
 * over requests and give no formula; the aggregation is the caller's.
 * All outputs are device fp32, row-major, written in full.
 */
typedef struct {
  int32_t layer;          /* 0 .. n_layers-1 */
  int32_t n_k;            /* 1 .. 16 */
  int32_t n_hours;        /* 0 .. 8192 */
  const float* event_age; /* required iff n_hours > 0 */
  float *recent, *topk;   /* required */
  float* hours;           /* required iff n_hours > 0 */
} llatte_attn_export;

/*
 * llatte_forward plus the statistics above, computed right after the
 * layer's attention from its stored queries and latent keys (scores in fp32).
 * Needs n_q > 0 and max_len <= LLATTE_EXPORT_MAX_LEN; LLATTE_ERR_ARG for bad
 * export arguments.  Asynchronous on `stream` like llatte_forward.
 */
#define LLATTE_EXPORT_MAX_LEN 4096
int llatte_forward_export(llatte_handle* handle, const void* values, const int64_t* offsets,
                          int32_t B, const void* context, const void* cand, float* out,
                          const llatte_attn_export* ex, void* stream);

/*
 * The forward pass of one llatte_batch (with the event ages, which the
 * timestamp code needs when d_time > 0); with ex != NULL it also computes the
 * attention statistics above (ex->event_age may then be the batch's).
 * Otherwise as llatte_forward.
 */
int llatte_forward_batch(llatte_handle* handle, const llatte_batch* batch, float* out,
                         const llatte_attn_export* ex, void* stream);

/*
 * Action tokenizer (appendix A.2 item 1 "Action Embeddings"): every history
 * event a_t = (tau_t, type_t, item_t, surface_t, meta_t) is embedded field by
 * field and projected to one token,
 *     x_t = MLP_act(E_type(type_t), E_item(item_t), E_surface(surface_t),
 *                   E_time(tau_t), E_meta(meta_t)) in R^d.
 * The pages name the parts and give no formula; the reading taken: each field
 * (the timestamp as its time-bucket id) is an integer id into its own table,
 * the embeddings are concatenated in field order, and
 *     x_t = W_a2 SiLU(W_a1 [e_1 ; ... ; e_F]),  no biases.
 * The tokens are the `values` rows of llatte_forward (same jagged layout).
 *
 *   n_fields        1 .. LLATTE_TOK_MAX_FIELDS tables
 *   rows[f]         rows of table f;  width[f] its embedding width, with
 *                   width[f] * element size a multiple of 16 bytes
 *                   (sum of widths = D_in, D_in * element size <= 2048 B)
 *   d_hid, d        hidden and token width (d * element size a multiple of 16)
 *   dtype           LLATTE_BF16 (tensor cores when D_in, d_hid are multiples
 *                   of 64 and d_hid, d of 64, else CUDA cores; for D_in = d =
 *                   256 and d_hid a multiple of 128 both products run in one
 *                   kernel whose output passes through fp16, so tokens must
 *                   stay below 65504 in magnitude) or LLATTE_FP32
 *   max_events      most events one call may tokenize (<= 65535 * 64)
 */
#define LLATTE_TOK_MAX_FIELDS 8
typedef struct {
  int32_t n_fields;
  int64_t rows[LLATTE_TOK_MAX_FIELDS];
  int32_t width[LLATTE_TOK_MAX_FIELDS];
  int32_t d_hid, d, dtype;
  int64_t max_events;
} llatte_tok_dims;

/*
 * Tokenizer parameters, in dtype, row-major:
 *   tables[f]  device [rows[f], width[f]], 16-byte aligned: NOT copied; the
 *              caller owns them and keeps them alive and unchanged while the
 *              tokenizer is used (embedding tables can be far larger than
 *              the rest of the model)
 *   W_a1       [d_hid, D_in]   W_a2 [d, d_hid]: copied at create (host memory
 *              if weights_on_device == 0, else device memory)
 */
typedef struct {
  const void* tables[LLATTE_TOK_MAX_FIELDS];
  const void *W_a1, *W_a2;
} llatte_tok_w;

typedef struct llatte_tokenizer llatte_tokenizer;

/* Create a tokenizer on the current device (synchronous); it owns copies of
 * W_a1, W_a2 and a workspace of max_events rows of D_in + d_hid elements. */
int llatte_tokenizer_create(llatte_tokenizer** tok, const llatte_tok_dims* dims,
                            const llatte_tok_w* weights, int weights_on_device);

/*
 * Tokens of n events, asynchronous on `stream`, no host synchronisation.
 *   ids     device int32 [n, n_fields], 4-byte aligned: event t's id per field
 *   n       0 <= n <= max_events (0 launches nothing)
 *   tokens  device [n, d] in dtype, 16-byte aligned: x_t for every event,
 *           ready to pass as llatte_forward's `values`
 * An id outside its table sets LLATTE_DEV_BAD_ID in the tokenizer's status
 * word and contributes a zero embedding (no out-of-range read).  Calls on
 * one tokenizer must not overlap in time (they share its workspace).
 */
int llatte_tokenize(llatte_tokenizer* tok, const int32_t* ids, int64_t n, void* tokens,
                    void* stream);

/* Synchronise the device, read the status word and clear it (as
 * llatte_get_status does for a forward handle). */
int llatte_tokenizer_get_status(llatte_tokenizer* tok, int32_t* device_status);

/* 1 when the two MLP_act GEMMs run on the tensor cores, 0 on CUDA cores. */
int llatte_tokenizer_uses_tensor_cores(const llatte_tokenizer* tok);

/* Free the tokenizer (synchronises its device); the tables stay the caller's. */
void llatte_tokenizer_destroy(llatte_tokenizer* tok);

/* Free the handle and everything it owns (synchronises its device). */
void llatte_destroy(llatte_handle* handle);

#ifdef __cplusplus
}
#endif

#endif /* LLATTE_H */
