// Action tokenizer: x_t = MLP_act(E_1(id_t1), ..., E_F(id_tF)) for every
// history event (LLaTTE notes, huaxiaozhuan.com, appendix A.2 item 1 "Action
// Embeddings"), read as x_t = W_a2 SiLU(W_a1 [e_1 ; ... ; e_F]) without biases.
//
//   embed_gather_kernel   E[t] = concatenated table rows of event t (HBM / L2
//                         bound: 16-byte vectors, four events per warp in flight)
//   then, for D_in = d = 256 in bf16, the fused FFN kernel on SM pairs
//   (W_a1 product, SiLU with the hidden layer kept in TMEM, W_a2 product,
//   bf16 rows stored into the caller's token rows); otherwise two GEMMs:
//   GEMM 1 (SiLU)         H = SiLU(E W_a1^T)      tcgen05 (bf16) or CUDA cores
//   GEMM 2 (store)        X = H W_a2^T            into the caller's token rows
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <new>

#include "common.cuh"
#include "internal.h"
#include "tc_ffn.h"
#include "tc_gemm.h"

using namespace llatte;

struct llatte_tokenizer {
  llatte_tok_dims dims;
  int device;
  int elem;
  int use_tc;
  int num_sms;
  int d_in;
  int bn1, bn2;
  int fused;                                   // both products in the fused FFN kernel
  const void* tables[LLATTE_TOK_MAX_FIELDS];   // caller-owned
  void* W_a1;                                  // [d_hid, d_in]
  void* W_a2;                                  // [d, d_hid]
  void* E;                                     // [max_events, d_in]
  void* H;                                     // [max_events, d_hid]
  int32_t* status;
  int64_t* n_dev;                              // events of the call in progress
  CUtensorMap tm_E, tm_H, tm_W1, tm_W2;
  CUtensorMap tm_W1h, tm_W2h;                  // fused kernel: 64- / 128-row weight boxes
};

namespace llatte {
namespace {

constexpr int kEmbedVecs = 4;            // 16-byte vectors per lane and event (row <= 2 KB)
constexpr int kGatherThreads = 256;
constexpr int kMaxBlockEvents = 128;     // events per block and round
constexpr int kGatherSmem = 65536;       // staged table vectors per block
constexpr int kLoadBatch = 4;            // vectors per thread in flight

struct EmbedArgs {
  const uint4* table[LLATTE_TOK_MAX_FIELDS];
  int64_t rows[LLATTE_TOK_MAX_FIELDS];
  int vec_off[LLATTE_TOK_MAX_FIELDS + 1];   // first vector of each field in an E row
  int n_fields, nvec;
  int block_events;                          // events per block and round
  const int32_t* ids;                        // [n, n_fields]
  int64_t n;
  int64_t* n_dev;                            // receives n (the fused kernel's row count)
  uint4* E;                                  // [n, nvec] vectors
  int32_t* status;
};

__device__ __forceinline__ int field_of(const EmbedArgs& a, int c) {
  int f = 0;
  while (f + 1 < a.n_fields && a.vec_off[f + 1] <= c) ++f;
  return f;
}

// E rows of a block of events.  Popular ids (Zipf item popularity) make many
// events read the same table row; read all at once by every SM, such a row's
// L2 lines serve the reads one after another.  So each block reads every
// distinct (field, id) of its events once: the first event with that id (its
// leader) loads the row into shared memory, and every event's E row is
// written from its leaders' copies.
__global__ void __launch_bounds__(kGatherThreads) embed_gather_kernel(EmbedArgs a) {
  extern __shared__ uint4 s_rows[];                     // [block_events][nvec]
  __shared__ int32_t s_id[kMaxBlockEvents * LLATTE_TOK_MAX_FIELDS];
  __shared__ int16_t s_lead[kMaxBlockEvents * LLATTE_TOK_MAX_FIELDS];
  __shared__ int8_t s_field[32 * kEmbedVecs];           // field of each vector of a row
  const int tid = threadIdx.x;
  const int F = a.n_fields, NV = a.nvec, EB = a.block_events;
  for (int c = tid; c < NV; c += kGatherThreads) s_field[c] = (int8_t)field_of(a, c);
  if (a.n_dev && blockIdx.x == 0 && tid == 0) *a.n_dev = a.n;
  int bad = 0;
  for (int64_t e0 = (int64_t)blockIdx.x * EB; e0 < a.n; e0 += (int64_t)gridDim.x * EB) {
    const int ne = (int)(a.n - e0 < EB ? a.n - e0 : EB);
    for (int i = tid; i < ne * F; i += kGatherThreads) s_id[i] = __ldg(a.ids + e0 * F + i);
    __syncthreads();
    // leader of (event e, field f): the first event of the block with the same id
    for (int i = tid; i < ne * F; i += kGatherThreads) {
      const int e = i / F, f = i - e * F, id = s_id[i];
      int l = e;
      for (int e2 = 0; e2 < e; ++e2)
        if (s_id[e2 * F + f] == id) { l = e2; break; }
      s_lead[i] = (int16_t)l;
    }
    __syncthreads();
    // leaders load their table vectors into their own slots, kLoadBatch in flight
    const int total = ne * NV;
    for (int v0 = tid; v0 < total; v0 += kGatherThreads * kLoadBatch) {
      uint4 buf[kLoadBatch];
      int slot[kLoadBatch];
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b) {
        const int v = v0 + b * kGatherThreads;
        slot[b] = -1;
        buf[b] = make_uint4(0, 0, 0, 0);
        if (v < total) {
          const int e = v / NV, c = v - e * NV, f = s_field[c];
          if (s_lead[e * F + f] == e) {
            slot[b] = v;
            const int64_t id = s_id[e * F + f];
            if (id >= 0 && id < a.rows[f]) {
              const int w = a.vec_off[f + 1] - a.vec_off[f];
              buf[b] = __ldg(a.table[f] + id * w + (c - a.vec_off[f]));
            } else {
              bad = 1;
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kLoadBatch; ++b)
        if (slot[b] >= 0) s_rows[slot[b]] = buf[b];
    }
    __syncthreads();
    // every event's row from its leaders' copies, coalesced 16-byte stores
    for (int v = tid; v < total; v += kGatherThreads) {
      const int e = v / NV, c = v - e * NV, f = s_field[c];
      const int l = s_lead[e * F + f];
      a.E[(e0 + e) * NV + c] = s_rows[l * NV + c];
    }
    __syncthreads();
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(a.status, LLATTE_DEV_BAD_ID);
}

// Events per block and round for rows of nvec 16-byte vectors.
int gather_block_events(int nvec) {
  const int fit = kGatherSmem / (nvec * 16);
  return fit < kMaxBlockEvents ? fit : kMaxBlockEvents;
}

cudaError_t launch_embed(const llatte_tokenizer* t, const int32_t* ids, int64_t n,
                         cudaStream_t s) {
  EmbedArgs a = {};
  const int F = t->dims.n_fields;
  a.n_fields = F;
  a.vec_off[0] = 0;
  for (int f = 0; f < F; ++f) {
    a.table[f] = (const uint4*)t->tables[f];
    a.rows[f] = t->dims.rows[f];
    a.vec_off[f + 1] = a.vec_off[f] + t->dims.width[f] * t->elem / 16;
  }
  a.nvec = a.vec_off[F];
  a.block_events = gather_block_events(a.nvec);
  a.ids = ids;
  a.n = n;
  a.n_dev = t->n_dev;
  a.E = (uint4*)t->E;
  a.status = t->status;
  const size_t smem = (size_t)a.block_events * a.nvec * 16;
  static uint64_t attr_devices = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_devices >> (dev & 63) & 1)) {
    cudaError_t e = cudaFuncSetAttribute(embed_gather_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kGatherSmem);
    if (e != cudaSuccess) return e;
    attr_devices |= 1ull << (dev & 63);
  }
  const int64_t groups = (n + a.block_events - 1) / a.block_events;
  const int64_t blocks = std::min<int64_t>(groups, (int64_t)t->num_sms * 3);
  embed_gather_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), kGatherThreads, smem, s>>>(a);
  return cudaGetLastError();
}

int check_tok_dims(const llatte_tok_dims* d) {
  if (!d) return LLATTE_ERR_ARG;
  if (d->n_fields < 1 || d->n_fields > LLATTE_TOK_MAX_FIELDS) return LLATTE_ERR_ARG;
  if (d->dtype != LLATTE_BF16 && d->dtype != LLATTE_FP32) return LLATTE_ERR_ARG;
  if (d->d <= 0 || d->d_hid <= 0 || d->max_events < 0) return LLATTE_ERR_ARG;
  const int e = d->dtype == LLATTE_BF16 ? 2 : 4;
  int64_t d_in = 0;
  for (int f = 0; f < d->n_fields; ++f) {
    if (d->rows[f] <= 0 || d->width[f] <= 0) return LLATTE_ERR_ARG;
    if ((d->width[f] * e) % 16 != 0) return LLATTE_ERR_UNSUPPORTED;   // 16-byte table rows
    d_in += d->width[f];
  }
  if (d_in * e > 32 * kEmbedVecs * 16) return LLATTE_ERR_UNSUPPORTED;  // E row <= 2 KB
  if ((d->d * e) % 16 != 0) return LLATTE_ERR_UNSUPPORTED;             // 16-byte token rows
  // CUDA-core GEMM grid: one 64-row block row per grid.y
  if (d->max_events > (int64_t)65535 * 64) return LLATTE_ERR_UNSUPPORTED;
  return LLATTE_OK;
}

void* dev_alloc(size_t bytes) {
  void* p = nullptr;
  if (cudaMalloc(&p, bytes ? bytes : 16) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace
}  // namespace llatte

extern "C" {

int llatte_tokenizer_create(llatte_tokenizer** out, const llatte_tok_dims* dims,
                            const llatte_tok_w* w, int weights_on_device) {
  if (!out) return LLATTE_ERR_ARG;
  *out = nullptr;
  int rc = check_tok_dims(dims);
  if (rc != LLATTE_OK) return rc;
  if (!w || !w->W_a1 || !w->W_a2) return LLATTE_ERR_ARG;
  for (int f = 0; f < dims->n_fields; ++f) {
    if (!w->tables[f] || ((uintptr_t)w->tables[f] & 15)) return LLATTE_ERR_ARG;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, w->tables[f]) != cudaSuccess ||
        (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)) {
      cudaGetLastError();
      return LLATTE_ERR_ARG;    // tables must be device memory
    }
  }
  llatte_tokenizer* t = new (std::nothrow) llatte_tokenizer();
  if (!t) return LLATTE_ERR_OOM;
  t->dims = *dims;
  t->elem = dims->dtype == LLATTE_BF16 ? 2 : 4;
  cudaGetDevice(&t->device);
  cudaDeviceGetAttribute(&t->num_sms, cudaDevAttrMultiProcessorCount, t->device);
  t->d_in = 0;
  for (int f = 0; f < dims->n_fields; ++f) {
    t->tables[f] = w->tables[f];
    t->d_in += dims->width[f];
  }
  const int64_t n = std::max<int64_t>(dims->max_events, 1);
  const size_t e = t->elem;
  auto fail = [&](int code) { llatte_tokenizer_destroy(t); return code; };
  t->W_a1 = dev_alloc(e * (size_t)dims->d_hid * t->d_in);
  t->W_a2 = dev_alloc(e * (size_t)dims->d * dims->d_hid);
  t->E = dev_alloc(e * (size_t)n * t->d_in);
  t->H = dev_alloc(e * (size_t)n * dims->d_hid);
  t->status = (int32_t*)dev_alloc(sizeof(int32_t));
  t->n_dev = (int64_t*)dev_alloc(sizeof(int64_t));
  if (!t->W_a1 || !t->W_a2 || !t->E || !t->H || !t->status || !t->n_dev)
    return fail(LLATTE_ERR_OOM);
  const cudaMemcpyKind kind = weights_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  if (cudaMemcpy(t->W_a1, w->W_a1, e * (size_t)dims->d_hid * t->d_in, kind) != cudaSuccess ||
      cudaMemcpy(t->W_a2, w->W_a2, e * (size_t)dims->d * dims->d_hid, kind) != cudaSuccess ||
      cudaMemset(t->status, 0, sizeof(int32_t)) != cudaSuccess ||
      cudaMemset(t->E, 0, e * (size_t)n * t->d_in) != cudaSuccess ||
      cudaMemset(t->H, 0, e * (size_t)n * dims->d_hid) != cudaSuccess)
    return fail(LLATTE_ERR_CUDA);
  // tensor cores when both GEMMs fit the tcgen05 kernel's tiles
  t->bn1 = dims->d_hid % 256 == 0 ? 256 : dims->d_hid % 128 == 0 ? 128 : 64;
  t->bn2 = dims->d % 256 == 0 ? 256 : dims->d % 128 == 0 ? 128 : 64;
  t->use_tc = dims->dtype == LLATTE_BF16 && tc_gemm_supported(t->bn1, TC_SILU, dims->d_hid, t->d_in) &&
              tc_gemm_supported(t->bn2, TC_STORE, dims->d, dims->d_hid);
  if (t->use_tc) {
    bool ok = make_tmap_bf16(&t->tm_E, t->E, n, t->d_in, 128) &&
              make_tmap_bf16(&t->tm_H, t->H, n, dims->d_hid, 128) &&
              make_tmap_bf16(&t->tm_W1, t->W_a1, dims->d_hid, t->d_in, std::min(t->bn1, 128)) &&
              make_tmap_bf16(&t->tm_W2, t->W_a2, dims->d, dims->d_hid, std::min(t->bn2, 128));
    if (!ok) t->use_tc = 0;
  }
  // the fused FFN kernel takes 256-wide inputs and outputs and a hidden width
  // that is a multiple of 128
  t->fused = t->use_tc && t->d_in == 256 && dims->d == 256 && ffn_tc_supported(256, dims->d_hid) &&
             make_tmap_bf16(&t->tm_W1h, t->W_a1, dims->d_hid, t->d_in, 64) &&
             make_tmap_bf16(&t->tm_W2h, t->W_a2, dims->d, dims->d_hid, 128);
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(LLATTE_ERR_CUDA);
  *out = t;
  return LLATTE_OK;
}

int llatte_tokenize(llatte_tokenizer* t, const int32_t* ids, int64_t n, void* tokens,
                    void* stream) {
  if (!t || n < 0 || n > t->dims.max_events) return LLATTE_ERR_ARG;
  if (n == 0) return LLATTE_OK;
  if (!ids || !tokens || ((uintptr_t)tokens & 15) || ((uintptr_t)ids & 3)) return LLATTE_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_embed(t, ids, n, s) != cudaSuccess) return LLATTE_ERR_CUDA;
  const llatte_tok_dims& D = t->dims;
  if (t->fused) {
    FfnTcParams f = {};
    f.M_dev = t->n_dev; f.M_cap = std::max<int64_t>(D.max_events, 1); f.F = D.d_hid;
    f.norm.mode = NORM_NONE; f.norm.dst = tokens; f.status = t->status;
    if (launch_ffn_pair(t->tm_E, t->tm_W1h, t->tm_W2h, f, t->num_sms, s) != cudaSuccess)
      return LLATTE_ERR_CUDA;
  } else if (t->use_tc) {
    TcGemmParams g1 = {};
    g1.M_host = n; g1.M_cap = n; g1.N = D.d_hid; g1.K = t->d_in;
    g1.D = (__nv_bfloat16*)t->H; g1.ldd = D.d_hid; g1.status = t->status;
    if (launch_tc_gemm(t->bn1, TC_SILU, t->tm_E, t->tm_W1, g1, t->num_sms, s) != cudaSuccess)
      return LLATTE_ERR_CUDA;
    TcGemmParams g2 = {};
    g2.M_host = n; g2.M_cap = n; g2.N = D.d; g2.K = D.d_hid;
    g2.D = (__nv_bfloat16*)tokens; g2.ldd = D.d; g2.status = t->status;
    if (launch_tc_gemm(t->bn2, TC_STORE, t->tm_H, t->tm_W2, g2, t->num_sms, s) != cudaSuccess)
      return LLATTE_ERR_CUDA;
  } else {
    GemmArgs g1 = {};
    g1.A = t->E; g1.lda = t->d_in; g1.W = t->W_a1; g1.D = t->H; g1.ldd = D.d_hid;
    g1.M_host = n; g1.M_max = n; g1.N = D.d_hid; g1.K = t->d_in; g1.epi = EPI_SILU;
    if (launch_gemm_simt(t->elem, t->elem, t->elem, g1, s) != cudaSuccess) return LLATTE_ERR_CUDA;
    GemmArgs g2 = {};
    g2.A = t->H; g2.lda = D.d_hid; g2.W = t->W_a2; g2.D = tokens; g2.ldd = D.d;
    g2.M_host = n; g2.M_max = n; g2.N = D.d; g2.K = D.d_hid; g2.epi = EPI_STORE;
    if (launch_gemm_simt(t->elem, t->elem, t->elem, g2, s) != cudaSuccess) return LLATTE_ERR_CUDA;
  }
  return LLATTE_OK;
}

int llatte_tokenizer_get_status(llatte_tokenizer* t, int32_t* device_status) {
  if (!t || !device_status) return LLATTE_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return LLATTE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, t->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(t->status, 0, sizeof(int32_t)) != cudaSuccess)
    return LLATTE_ERR_CUDA;
  *device_status = v;
  return v ? LLATTE_ERR_DEVICE : LLATTE_OK;
}

int llatte_tokenizer_uses_tensor_cores(const llatte_tokenizer* t) {
  return t ? t->use_tc : LLATTE_ERR_ARG;
}

void llatte_tokenizer_destroy(llatte_tokenizer* t) {
  if (!t) return;
  cudaDeviceSynchronize();
  cudaFree(t->W_a1);
  cudaFree(t->W_a2);
  cudaFree(t->E);
  cudaFree(t->H);
  cudaFree(t->status);
  cudaFree(t->n_dev);
  delete t;
}

}  // extern "C"
