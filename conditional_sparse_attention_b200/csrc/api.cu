// C ABI entry points: argument validation, context scratch, conditional capture, graphs,
// error reporting.  Every compute step is one of the kernels in attention.cu, head.cu,
// commit.cu and glue.cu.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

namespace oda {

oda_status prepare_head_kernel();

static thread_local char g_msg[512] = "";

oda_status set_error(oda_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return s;
}

oda_status check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ODA_OK;
  return set_error(ODA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

oda_status validate_attention_config(const oda_config& c, const char* who) {
  if (c.batch < 1 || c.batch > ODA_MAX_BATCH)
    return set_error(ODA_ERR_UNSUPPORTED, "%s: batch must be 1..%d", who, ODA_MAX_BATCH);
  if (c.n_q_heads < 1 || c.n_kv_heads < 1 || c.n_q_heads % c.n_kv_heads != 0 ||
      c.n_q_heads / c.n_kv_heads > 8)
    return set_error(ODA_ERR_UNSUPPORTED, "%s: need Hq %% Hkv == 0 and Hq/Hkv <= 8", who);
  if (c.head_dim != 128) return set_error(ODA_ERR_UNSUPPORTED, "%s: head_dim must be 128", who);
  if (c.page_size != 16) return set_error(ODA_ERR_UNSUPPORTED, "%s: page_size must be 16", who);
  if (c.max_pages < 1 || (int64_t)c.max_pages * 16 > INT32_MAX - 1)
    return set_error(ODA_ERR_INVALID_ARG, "%s: max_pages out of range", who);
  if (c.sinks < 0 || c.sinks > 16) return set_error(ODA_ERR_UNSUPPORTED, "%s: sinks must be 0..16", who);
  if (c.window < 1) return set_error(ODA_ERR_INVALID_ARG, "%s: window must be >= 1", who);
  if (c.deterministic != 0 && c.deterministic != 1)
    return set_error(ODA_ERR_INVALID_ARG, "%s: deterministic must be 0 or 1", who);
  return ODA_OK;
}

__global__ void set_condition_kernel(cudaGraphConditionalHandle h, const int32_t* any_flag) {
  grid_dependency_wait();   // any_flag comes from the kernel before (programmatic launch)
  cudaGraphSetConditional(h, *any_flag != 0 ? 1u : 0u);
}

// Diagnostic: one bounded wait that can never complete, through the same helpers the kernels
// use.  which = 0: an mbarrier that nothing arrives on (the copy-ring waits); which = 1: a
// grid barrier whose target is one CTA more than the grid (the fused head's phase barrier).
// The wait gives up after limit_ns and sets ODA_DEVERR_WAIT_TIMEOUT; the counter is handed
// back to zero before the kernel returns.
__global__ void wait_probe_kernel(int which, uint64_t limit_ns, int32_t* ctr, int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  bool ok;
  if (which == 0) {
    ok = mbar_wait_bounded(&bar, 0u, limit_ns);
  } else {
    ok = grid_barrier_bounded(ctr, (int)gridDim.x + 1, limit_ns);
    atomicSub(ctr, 1);
  }
  if (!ok) atomicOr(err, ODA_DEVERR_WAIT_TIMEOUT);
}

oda_status launch_set_condition(cudaGraphConditionalHandle h, const int32_t* any_flag,
                                bool overlap, cudaStream_t stream) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(1);
  lc.blockDim = dim3(1);
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = overlap ? 1 : 0;
  return check_cuda(cudaLaunchKernelEx(&lc, set_condition_kernel, h, any_flag),
                    "set-condition launch");
}

}  // namespace oda

using oda::check_cuda;
using oda::set_error;

struct oda_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

namespace {

template <class T>
oda_status dev_alloc(T** p, size_t n, const char* what) {
  *p = nullptr;
  if (n == 0) n = 1;
  return check_cuda(cudaMalloc(reinterpret_cast<void**>(p), n * sizeof(T)), what);
}

void free_ctx(oda_ctx* c) {
  if (!c) return;
  void* ptrs[] = {c->part_o, c->part_ml, c->attn_cnt, c->err, c->head_part, c->head_ss,
                  c->head_cnt, c->head_u, c->head_f, c->head_act, c->glue_x, c->glue_ss,
                  c->glue_cnt, c->bb_part, c->bb_cnt};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  if (c->body_stream) cudaStreamDestroy(c->body_stream);
  delete c;
}

bool stream_capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return false;
  return cs == cudaStreamCaptureStatusActive;
}

}  // namespace

extern "C" {

int32_t oda_version(void) { return ODA_VERSION_MAJOR * 100 + ODA_VERSION_MINOR; }

const char* oda_status_string(oda_status s) {
  switch (s) {
    case ODA_OK: return "ODA_OK";
    case ODA_ERR_INVALID_ARG: return "ODA_ERR_INVALID_ARG";
    case ODA_ERR_UNSUPPORTED: return "ODA_ERR_UNSUPPORTED";
    case ODA_ERR_CUDA: return "ODA_ERR_CUDA";
    case ODA_ERR_DEVICE: return "ODA_ERR_DEVICE";
    case ODA_ERR_STATE: return "ODA_ERR_STATE";
  }
  return "ODA_ERR_UNKNOWN";
}

const char* oda_last_error(void) { return oda::g_msg; }

oda_status oda_create(const oda_config* cfg, oda_ctx** out) {
  if (!out) return set_error(ODA_ERR_INVALID_ARG, "create: out is NULL");
  *out = nullptr;
  if (!cfg) return set_error(ODA_ERR_INVALID_ARG, "create: cfg is NULL");
  const oda_config& c = *cfg;
  oda_status vs = oda::validate_attention_config(c, "create");
  if (vs != ODA_OK) return vs;
  if (c.head_in_dim < 512 || c.head_in_dim > 8192 || c.head_in_dim % 512 != 0)
    return set_error(ODA_ERR_UNSUPPORTED, "create: head_in_dim must be a multiple of 512 in 512..8192");
  if (c.overlap_layers != 0 && c.overlap_layers != 1)
    return set_error(ODA_ERR_INVALID_ARG, "create: overlap_layers must be 0 or 1");

  oda_ctx* x = new oda_ctx();
  x->cfg = c;
  x->g = c.n_q_heads / c.n_kv_heads;
  oda_status st = check_cuda(cudaGetDevice(&x->device), "cudaGetDevice");
  if (st == ODA_OK)
    st = check_cuda(cudaDeviceGetAttribute(&x->n_sms, cudaDevAttrMultiProcessorCount, x->device),
                    "cudaDeviceGetAttribute");
  if (st == ODA_OK) st = oda::prepare_attention_kernel(x->g, x->n_sms, x->attn_ctas);
  if (st == ODA_OK) st = oda::prepare_head_kernel();
  if (st != ODA_OK) {
    free_ctx(x);
    return st;
  }
  const int64_t B = c.batch, Hkv = c.n_kv_heads, D = c.head_in_dim;
  x->n_slots = (int)(std::max(x->attn_ctas[0], x->attn_ctas[1]) + B * Hkv);
  const int64_t ms = x->n_slots;
  const int gch = oda::glue_chunks(c.head_in_dim);
  st = dev_alloc(&x->part_o, (size_t)ms * x->g * 128, "cudaMalloc(partials)");
  if (st == ODA_OK) st = dev_alloc(&x->part_ml, (size_t)ms * x->g * 2, "cudaMalloc(partials)");
  if (st == ODA_OK) st = dev_alloc(&x->attn_cnt, (size_t)2 * B * Hkv, "cudaMalloc(counters)");
  if (st == ODA_OK) st = dev_alloc(&x->err, 1, "cudaMalloc(error word)");
  if (st == ODA_OK) st = dev_alloc(&x->head_part, oda::head_part_floats((int)B, (int)D), "cudaMalloc(head)");
  if (st == ODA_OK) st = dev_alloc(&x->head_ss, oda::head_ss_floats((int)B, (int)D), "cudaMalloc(head)");
  if (st == ODA_OK) st = dev_alloc(&x->head_cnt, (size_t)oda::head_counter_count((int)D), "cudaMalloc(head)");
  if (st == ODA_OK) st = dev_alloc(&x->head_u, (size_t)3 * B * 1024, "cudaMalloc(head)");
  if (st == ODA_OK) st = dev_alloc(&x->head_f, (size_t)3 * B * 1024, "cudaMalloc(head)");
  if (st == ODA_OK) st = dev_alloc(&x->head_act, (size_t)B * 2048, "cudaMalloc(head)");
  if (st == ODA_OK) st = dev_alloc(&x->glue_x, (size_t)B * D, "cudaMalloc(glue)");
  if (st == ODA_OK) st = dev_alloc(&x->glue_ss, (size_t)B * gch, "cudaMalloc(glue)");
  if (st == ODA_OK) st = dev_alloc(&x->glue_cnt, (size_t)2 * B, "cudaMalloc(glue)");
  // backbone projections: split-K partials (up to 1M floats) and per-tile counters
  x->bb_part_floats = (size_t)1 << 20;
  x->bb_cnt_n = 4096;
  if (st == ODA_OK) st = dev_alloc(&x->bb_part, x->bb_part_floats, "cudaMalloc(backbone)");
  if (st == ODA_OK) st = dev_alloc(&x->bb_cnt, (size_t)x->bb_cnt_n, "cudaMalloc(backbone)");
  if (st == ODA_OK) st = check_cuda(cudaMemset(x->bb_cnt, 0, x->bb_cnt_n * sizeof(int32_t)), "cudaMemset");
  if (st == ODA_OK) st = check_cuda(cudaMemset(x->attn_cnt, 0, 2 * B * Hkv * sizeof(int32_t)), "cudaMemset");
  if (st == ODA_OK) st = check_cuda(cudaMemset(x->err, 0, sizeof(int32_t)), "cudaMemset");
  if (st == ODA_OK)
    st = check_cuda(cudaMemset(x->head_cnt, 0, oda::head_counter_count((int)D) * sizeof(int32_t)),
                    "cudaMemset");
  if (st == ODA_OK) st = check_cuda(cudaMemset(x->glue_cnt, 0, 2 * B * sizeof(int32_t)), "cudaMemset");
  if (st == ODA_OK)
    st = check_cuda(cudaStreamCreateWithFlags(&x->body_stream, cudaStreamNonBlocking),
                    "cudaStreamCreate");
  if (st == ODA_OK) st = check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  if (st != ODA_OK) {
    free_ctx(x);
    return st;
  }
  *out = x;
  return ODA_OK;
}

oda_status oda_destroy(oda_ctx* ctx) {
  if (!ctx) return ODA_OK;
  cudaDeviceSynchronize();
  free_ctx(ctx);
  return ODA_OK;
}

oda_status oda_attend_local(oda_ctx* ctx, const oda_kv_layer* layer, const int32_t* page_table,
                            const int32_t* pos, const void* q, const void* k_new,
                            const void* v_new, float* out, cudaStream_t stream) {
  if (!ctx || !layer) return set_error(ODA_ERR_INVALID_ARG, "attend_local: ctx or layer is NULL");
  const oda::KvPool pool{0, layer->k, layer->v, layer->n_pages};
  return oda::launch_attention(ctx, pool, page_table, pos, nullptr, q, k_new, v_new, out, 0, stream);
}

oda_status oda_attend_full_if(oda_ctx* ctx, const oda_kv_layer* layer, const int32_t* page_table,
                              const int32_t* pos, const int32_t* flag, const void* q,
                              const void* k_new, const void* v_new, float* out,
                              cudaStream_t stream) {
  if (!ctx || !layer) return set_error(ODA_ERR_INVALID_ARG, "attend_full_if: ctx or layer is NULL");
  const oda::KvPool pool{0, layer->k, layer->v, layer->n_pages};
  return oda::launch_attention(ctx, pool, page_table, pos, flag, q, k_new, v_new, out, 1, stream);
}

oda_status oda_attend_local_fp8(oda_ctx* ctx, const oda_kv8_layer* layer, const int32_t* page_table,
                                const int32_t* pos, const void* q, const void* k_new,
                                const void* v_new, float* out, cudaStream_t stream) {
  if (!ctx || !layer) return set_error(ODA_ERR_INVALID_ARG, "attend_local_fp8: ctx or layer is NULL");
  const oda::KvPool pool{1, layer->kv, nullptr, layer->n_pages};
  return oda::launch_attention(ctx, pool, page_table, pos, nullptr, q, k_new, v_new, out, 0, stream);
}

oda_status oda_attend_full_if_fp8(oda_ctx* ctx, const oda_kv8_layer* layer, const int32_t* page_table,
                                  const int32_t* pos, const int32_t* flag, const void* q,
                                  const void* k_new, const void* v_new, float* out,
                                  cudaStream_t stream) {
  if (!ctx || !layer) return set_error(ODA_ERR_INVALID_ARG, "attend_full_if_fp8: ctx or layer is NULL");
  const oda::KvPool pool{1, layer->kv, nullptr, layer->n_pages};
  return oda::launch_attention(ctx, pool, page_table, pos, flag, q, k_new, v_new, out, 1, stream);
}

oda_status oda_kv8_pack(const oda_kv_layer* src, const oda_kv8_layer* dst, int32_t n_kv_heads,
                        cudaStream_t stream) {
  return oda::launch_kv8_pack(src, dst, n_kv_heads, stream);
}

oda_status oda_attend_full_if_noalloc(const oda_config* cfg, const oda_kv_layer* layer,
                                      const int32_t* page_table, const int32_t* pos,
                                      const int32_t* flag, const void* q, const void* k_new,
                                      const void* v_new, float* out, int32_t* device_error,
                                      cudaStream_t stream) {
  return oda::launch_attention_noalloc(cfg, layer, page_table, pos, flag, q, k_new, v_new, out,
                                       device_error, stream);
}

oda_status oda_index_positions(oda_ctx* ctx, int32_t mode, const int32_t* pos, const int32_t* flag,
                               int32_t* positions, int32_t cap, int32_t* counts,
                               cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "index_positions: ctx is NULL");
  return oda::launch_index_positions(ctx, mode, pos, flag, positions, cap, counts, stream);
}

oda_status oda_recall_score(oda_ctx* ctx, const oda_head_weights* w, const float* h_prev,
                            const float* emb, const float* h_loc, const int32_t* sched,
                            float* score, int32_t* flag, int32_t* any_flag, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "recall_score: ctx is NULL");
  ctx->prev_attention = false;
  return oda::launch_recall_head(ctx, w, h_prev, emb, h_loc, sched, score, flag, any_flag, stream);
}

oda_status oda_recall_plan(oda_ctx* ctx, int32_t* tile, int32_t* groups, int32_t* ring) {
  if (!ctx || !tile || !groups || !ring) return set_error(ODA_ERR_INVALID_ARG, "recall_plan: null argument");
  return oda::recall_head_plan(ctx, tile, groups, ring);
}

size_t oda_recall_grad_workspace_bytes(int32_t batch, int32_t head_in_dim) {
  if (batch < 1 || head_in_dim < 1) return 0;
  return oda::recall_grad_workspace_bytes(batch, head_in_dim);
}

oda_status oda_recall_grad(const oda_head_weights* w, const oda_head_grads* grad, int32_t batch,
                           int32_t head_in_dim, const float* h_prev, const float* emb,
                           const float* h_loc, const float* p_full, const float* p_local,
                           const int32_t* valid, float lambda, float* loss, float* q, float* y,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!(lambda >= 0.f)) return set_error(ODA_ERR_INVALID_ARG, "recall_grad: lambda must be >= 0");
  return oda::launch_recall_grad(w, grad, batch, head_in_dim, h_prev, emb, h_loc, p_full, p_local,
                                 valid, lambda, loss, q, y, workspace, workspace_bytes, stream);
}

oda_status oda_commit(oda_ctx* ctx, const oda_kv_layer* layers, int32_t n_layers,
                      const int32_t* page_table, int32_t* pos, const int32_t* flag,
                      const void* k_stage_local, const void* v_stage_local,
                      const void* k_stage_full, const void* v_stage_full,
                      const float* h_local, const float* h_full, float* h_prev,
                      cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "commit: ctx is NULL");
  if (!layers || n_layers < 1 || n_layers > ODA_MAX_LAYERS)
    return set_error(ODA_ERR_INVALID_ARG, "commit: n_layers must be 1..%d", ODA_MAX_LAYERS);
  ctx->prev_attention = false;
  oda::KvPool pools[ODA_MAX_LAYERS];
  for (int l = 0; l < n_layers; ++l) pools[l] = {0, layers[l].k, layers[l].v, layers[l].n_pages};
  return oda::launch_commit(ctx, pools, n_layers, page_table, pos, flag, k_stage_local,
                            v_stage_local, k_stage_full, v_stage_full, h_local, h_full, h_prev,
                            stream);
}

oda_status oda_commit_fp8(oda_ctx* ctx, const oda_kv8_layer* layers, int32_t n_layers,
                          const int32_t* page_table, int32_t* pos, const int32_t* flag,
                          const void* k_stage_local, const void* v_stage_local,
                          const void* k_stage_full, const void* v_stage_full,
                          const float* h_local, const float* h_full, float* h_prev,
                          cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "commit_fp8: ctx is NULL");
  if (!layers || n_layers < 1 || n_layers > ODA_MAX_LAYERS)
    return set_error(ODA_ERR_INVALID_ARG, "commit_fp8: n_layers must be 1..%d", ODA_MAX_LAYERS);
  ctx->prev_attention = false;
  oda::KvPool pools[ODA_MAX_LAYERS];
  for (int l = 0; l < n_layers; ++l) pools[l] = {1, layers[l].kv, nullptr, layers[l].n_pages};
  return oda::launch_commit(ctx, pools, n_layers, page_table, pos, flag, k_stage_local,
                            v_stage_local, k_stage_full, v_stage_full, h_local, h_full, h_prev,
                            stream);
}

oda_status oda_snapshot(oda_ctx* ctx, const oda_state* live, const oda_state* snap,
                        cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "snapshot: ctx is NULL");
  ctx->prev_attention = false;
  return oda::launch_state_copy(live, snap, ctx->cfg.batch, nullptr, stream);
}

oda_status oda_restore(oda_ctx* ctx, const int32_t* flag, const oda_state* snap,
                       const oda_state* live, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "restore: ctx is NULL");
  if (!flag) return set_error(ODA_ERR_INVALID_ARG, "restore: flag is NULL");
  ctx->prev_attention = false;
  return oda::launch_state_copy(snap, live, ctx->cfg.batch, flag, stream);
}

oda_status oda_glue_hidden(oda_ctx* ctx, const float* emb, const float* terms, int32_t n_terms,
                           const int32_t* flag, float* h, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "glue_hidden: ctx is NULL");
  ctx->prev_attention = false;
  return oda::launch_glue_hidden(ctx, emb, terms, n_terms, flag, h, stream);
}

oda_status oda_glue_gdn(oda_ctx* ctx, const oda_state* st, int32_t layer, const float* c,
                        const float* v, const float* alpha, const float* beta,
                        const float* taps, const int32_t* flag, float* o, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "glue_gdn: ctx is NULL");
  ctx->prev_attention = false;
  return oda::launch_glue_gdn(ctx, st, st, layer, c, v, alpha, beta, taps, flag, o, stream);
}

oda_status oda_glue_gdn_step(oda_ctx* ctx, const oda_state* src, const oda_state* dst,
                             int32_t layer, const float* c, const float* v, const float* alpha,
                             const float* beta, const float* taps, const int32_t* flag, float* o,
                             cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "glue_gdn_step: ctx is NULL");
  ctx->prev_attention = false;
  return oda::launch_glue_gdn(ctx, src, dst, layer, c, v, alpha, beta, taps, flag, o, stream);
}

oda_status oda_bb_begin(oda_ctx* ctx, const float* emb, float* x, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_begin: ctx is NULL");
  return oda::launch_bb_begin(ctx, emb, x, stream);
}

oda_status oda_bb_qkv(oda_ctx* ctx, const oda_bb_layer* layer, const float* x, void* q,
                      void* k_new, void* v_new, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_qkv: ctx is NULL");
  return oda::launch_bb_qkv(ctx, layer, x, q, k_new, v_new, stream);
}

oda_status oda_bb_attn_out(oda_ctx* ctx, const oda_bb_layer* layer, const float* o, float* x,
                           cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_attn_out: ctx is NULL");
  return oda::launch_bb_attn_out(ctx, layer, o, x, stream);
}

oda_status oda_bb_mlp(oda_ctx* ctx, const oda_bb_layer* layer, float* x, void* act,
                      cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_mlp: ctx is NULL");
  return oda::launch_bb_mlp(ctx, layer, x, act, stream);
}

oda_status oda_bb_post_attention(oda_ctx* ctx, const oda_bb_layer* layer, const oda_bb_layer* next,
                                 const float* o, float* x, void* act, void* q, void* k_new,
                                 void* v_new, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_post_attention: ctx is NULL");
  return oda::launch_bb_post(ctx, layer, next, o, x, act, q, k_new, v_new, stream);
}

oda_status oda_bb_pack_weight(oda_ctx* ctx, const void* src, int32_t rows, int32_t cols, void* dst,
                              cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_pack_weight: ctx is NULL");
  return oda::launch_bb_pack_weight(ctx, src, rows, cols, dst, stream);
}

oda_status oda_bb_final_norm(oda_ctx* ctx, const float* gamma, const float* x, float* h,
                             cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_final_norm: ctx is NULL");
  return oda::launch_bb_final_norm(ctx, gamma, x, h, stream);
}

oda_status oda_bb_lm_head(oda_ctx* ctx, const void* embed, int32_t vocab, const float* h,
                          float* logits, int32_t* token, float* next_emb, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_lm_head: ctx is NULL");
  return oda::launch_bb_lm_head(ctx, embed, vocab, h, logits, token, next_emb, stream);
}

oda_status oda_bb_embed(oda_ctx* ctx, const void* embed, int32_t vocab, int32_t* token,
                        float* emb, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "bb_embed: ctx is NULL");
  return oda::launch_bb_embed(ctx, embed, vocab, token, emb, stream);
}

oda_status oda_cond_begin(oda_ctx* ctx, cudaStream_t stream, const int32_t* any_flag,
                          cudaStream_t* body_stream) {
  if (!ctx || !any_flag || !body_stream)
    return set_error(ODA_ERR_INVALID_ARG, "cond_begin: null argument");
  if (ctx->cond_open) return set_error(ODA_ERR_STATE, "cond_begin: a conditional is already open");
  ctx->prev_attention = false;
  if (!stream_capturing(stream)) {
    ctx->cond_open = true;
    ctx->cond_parent = nullptr;
    *body_stream = stream;
    return ODA_OK;
  }
  cudaStreamCaptureStatus cs;
  cudaGraph_t graph = nullptr;
  const cudaGraphNode_t* deps = nullptr;
  size_t nd = 0;
  oda_status st = check_cuda(cudaStreamGetCaptureInfo(stream, &cs, nullptr, &graph, &deps, &nd),
                             "cudaStreamGetCaptureInfo");
  if (st != ODA_OK) return st;
  cudaGraphConditionalHandle h;
  st = check_cuda(cudaGraphConditionalHandleCreate(&h, graph, 0, cudaGraphCondAssignDefault),
                  "cudaGraphConditionalHandleCreate");
  if (st != ODA_OK) return st;
  st = oda::launch_set_condition(h, any_flag, ctx->cfg.overlap_layers != 0, stream);
  if (st != ODA_OK) return st;
  st = check_cuda(cudaStreamGetCaptureInfo(stream, &cs, nullptr, &graph, &deps, &nd),
                  "cudaStreamGetCaptureInfo");
  if (st != ODA_OK) return st;
  cudaGraphNodeParams np = {cudaGraphNodeTypeConditional};
  np.conditional.handle = h;
  np.conditional.type = cudaGraphCondTypeIf;
  np.conditional.size = 1;
  cudaGraphNode_t node;
  st = check_cuda(cudaGraphAddNode(&node, graph, deps, nd, &np), "cudaGraphAddNode(conditional)");
  if (st != ODA_OK) return st;
  cudaGraph_t body = np.conditional.phGraph_out[0];
  st = check_cuda(cudaStreamUpdateCaptureDependencies(stream, &node, 1,
                                                      cudaStreamSetCaptureDependencies),
                  "cudaStreamUpdateCaptureDependencies");
  if (st != ODA_OK) return st;
  st = check_cuda(cudaStreamBeginCaptureToGraph(ctx->body_stream, body, nullptr, nullptr, 0,
                                                cudaStreamCaptureModeRelaxed),
                  "cudaStreamBeginCaptureToGraph");
  if (st != ODA_OK) return st;
  ctx->cond_open = true;
  ctx->cond_parent = stream;
  *body_stream = ctx->body_stream;
  return ODA_OK;
}

oda_status oda_cond_end(oda_ctx* ctx, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "cond_end: ctx is NULL");
  if (!ctx->cond_open) return set_error(ODA_ERR_STATE, "cond_end: no open conditional");
  ctx->cond_open = false;
  ctx->prev_attention = false;
  if (ctx->cond_parent == nullptr) return ODA_OK;
  if (ctx->cond_parent != stream)
    return set_error(ODA_ERR_STATE, "cond_end: stream differs from the one given to cond_begin");
  ctx->cond_parent = nullptr;
  cudaGraph_t g = nullptr;
  return check_cuda(cudaStreamEndCapture(ctx->body_stream, &g), "cudaStreamEndCapture(body)");
}

oda_status oda_graph_begin(cudaStream_t stream) {
  return check_cuda(cudaStreamBeginCapture(stream, cudaStreamCaptureModeRelaxed),
                    "cudaStreamBeginCapture");
}

oda_status oda_graph_end(cudaStream_t stream, oda_graph** out) {
  if (!out) return set_error(ODA_ERR_INVALID_ARG, "graph_end: out is NULL");
  *out = nullptr;
  oda_graph* g = new oda_graph();
  oda_status st = check_cuda(cudaStreamEndCapture(stream, &g->graph), "cudaStreamEndCapture");
  if (st == ODA_OK)
    st = check_cuda(cudaGraphInstantiate(&g->exec, g->graph, 0), "cudaGraphInstantiate");
  if (st != ODA_OK) {
    if (g->graph) cudaGraphDestroy(g->graph);
    delete g;
    return st;
  }
  *out = g;
  return ODA_OK;
}

oda_status oda_graph_launch(oda_graph* g, cudaStream_t stream) {
  if (!g) return set_error(ODA_ERR_INVALID_ARG, "graph_launch: graph is NULL");
  return check_cuda(cudaGraphLaunch(g->exec, stream), "cudaGraphLaunch");
}

oda_status oda_graph_destroy(oda_graph* g) {
  if (!g) return ODA_OK;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  delete g;
  return ODA_OK;
}

oda_status oda_probe_wait(oda_ctx* ctx, int32_t which, int64_t limit_ns, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "probe_wait: ctx is NULL");
  if ((which != 0 && which != 1) || limit_ns < 1000 || limit_ns > 1000000000)
    return set_error(ODA_ERR_INVALID_ARG, "probe_wait: which must be 0 or 1, limit 1 us .. 1 s");
  ctx->prev_attention = false;
  // the fused head's barrier counter: zero between launches, and back to zero after the probe
  oda::wait_probe_kernel<<<1, 1, 0, stream>>>(which, (uint64_t)limit_ns, ctx->head_cnt, ctx->err);
  return check_cuda(cudaGetLastError(), "probe_wait launch");
}

oda_status oda_get_error(oda_ctx* ctx, int32_t* device_error) {
  if (!ctx || !device_error) return set_error(ODA_ERR_INVALID_ARG, "get_error: null argument");
  oda_status st = check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  if (st != ODA_OK) return st;
  st = check_cuda(cudaMemcpy(device_error, ctx->err, sizeof(int32_t), cudaMemcpyDeviceToHost),
                  "cudaMemcpy(error word)");
  if (st != ODA_OK) return st;
  if (*device_error != 0)
    return set_error(ODA_ERR_DEVICE, "device error word 0x%x", (unsigned)*device_error);
  return ODA_OK;
}

oda_status oda_clear_error(oda_ctx* ctx, cudaStream_t stream) {
  if (!ctx) return set_error(ODA_ERR_INVALID_ARG, "clear_error: ctx is NULL");
  ctx->prev_attention = false;
  return check_cuda(cudaMemsetAsync(ctx->err, 0, sizeof(int32_t), stream), "cudaMemsetAsync");
}

}  // extern "C"
