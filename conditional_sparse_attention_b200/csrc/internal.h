// Internal declarations shared by the library's translation units (not installed).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "oda.h"
#include "oda_glue.h"
#include "oda_backbone.h"

struct oda_ctx {
  oda_config cfg;
  int device = 0;
  int n_sms = 0;
  int g = 1;
  // split-KV attention scratch
  int attn_ctas[2] = {0, 0};  // persistent grid size of the full-set kernel: bf16, fp8 pages
  int n_slots = 0;            // partial slots: max(attn_ctas) + B*Hkv
  float* part_o = nullptr;    // [n_slots][g][128]
  float* part_ml = nullptr;   // [n_slots][g][2]
  int32_t* attn_cnt = nullptr;  // [2][B*Hkv] completion and chunk-claim counters (self-resetting)
  int32_t* err = nullptr;       // sticky device error word
  // recall-head scratch
  float* head_part = nullptr;   // split-K partial sums, largest phase
  float* head_ss = nullptr;     // partial sums of squares of the tower inputs
  int32_t* head_cnt = nullptr;  // per row-block completion counters + final counter
  float* head_u = nullptr;      // [3][B][1024]
  float* head_f = nullptr;      // [3][B][1024]: fusion output and the two block outputs
  float* head_act = nullptr;    // [B][2048]
  // synthetic-backbone scratch: split-K partial sums and per-tile completion counters
  float* bb_part = nullptr;
  size_t bb_part_floats = 0;
  int32_t* bb_cnt = nullptr;
  int bb_cnt_n = 0;
  // glue scratch
  float* glue_x = nullptr;      // [B][D]
  float* glue_ss = nullptr;     // [B][chunks]
  int32_t* glue_cnt = nullptr;  // [B]
  // conditional capture
  cudaStream_t body_stream = nullptr;
  cudaStream_t cond_parent = nullptr;
  bool cond_open = false;
  // true when the last kernel this context launched was an attention kernel: the next
  // attention launch may then overlap it (programmatic dependent launch)
  bool prev_attention = false;
  void* alloc_base = nullptr;
};

namespace oda {

oda_status set_error(oda_status s, const char* fmt, ...);
oda_status check_cuda(cudaError_t e, const char* what);
// Shape checks shared by oda_create and the allocation-free attention entry point: every field
// of oda_config except head_in_dim, theta and overlap_layers.
oda_status validate_attention_config(const oda_config& c, const char* who);

// Where one layer's cached pages live: fmt 0 = bf16 K and V pools (k, v), fmt 1 = fp8 page
// blocks (k; v unused).
struct KvPool {
  int fmt;
  const void* k;
  const void* v;
  int64_t n_pages;
};

// attention.cu
oda_status launch_attention(oda_ctx* ctx, const KvPool& pool, const int32_t* page_table,
                            const int32_t* pos, const int32_t* flag, const void* q,
                            const void* k_new, const void* v_new, float* out, int mode,
                            cudaStream_t stream);
oda_status launch_index_positions(oda_ctx* ctx, int mode, const int32_t* pos, const int32_t* flag,
                                  int32_t* positions, int32_t cap, int32_t* counts,
                                  cudaStream_t stream);
int attention_smem_bytes(int g);
oda_status prepare_attention_kernel(int g, int n_sms, int* ctas /* [2] */);
oda_status launch_attention_noalloc(const oda_config* cfg, const oda_kv_layer* layer,
                                    const int32_t* page_table, const int32_t* pos,
                                    const int32_t* flag, const void* q, const void* k_new,
                                    const void* v_new, float* out, int32_t* device_error,
                                    cudaStream_t stream);

// head.cu
oda_status launch_recall_head(oda_ctx* ctx, const oda_head_weights* w, const float* h_prev,
                              const float* emb, const float* h_loc, const int32_t* sched,
                              float* score, int32_t* flag, int32_t* any_flag, cudaStream_t s);
oda_status recall_head_plan(oda_ctx* ctx, int32_t* tile, int32_t* groups, int32_t* ring);
size_t head_part_floats(int B, int D);
size_t head_ss_floats(int B, int D);
int head_counter_count(int D);

// head_grad.cu
size_t recall_grad_workspace_bytes(int B, int D);
oda_status launch_recall_grad(const oda_head_weights* w, const oda_head_grads* gr, int B, int D,
                              const float* h_prev, const float* emb, const float* h_loc,
                              const float* p_full, const float* p_local, const int32_t* valid,
                              float lam, float* loss, float* q, float* y, void* workspace,
                              size_t workspace_bytes, cudaStream_t s);

// commit.cu
oda_status launch_kv8_pack(const oda_kv_layer* src, const oda_kv8_layer* dst, int32_t n_kv_heads,
                           cudaStream_t stream);
oda_status launch_commit(oda_ctx* ctx, const KvPool* layers, int32_t n_layers,
                         const int32_t* page_table, int32_t* pos, const int32_t* flag,
                         const void* ksl, const void* vsl, const void* ksf, const void* vsf,
                         const float* h_local, const float* h_full, float* h_prev,
                         cudaStream_t stream);
oda_status launch_state_copy(const oda_state* src, const oda_state* dst, int B,
                             const int32_t* flag, cudaStream_t stream);

// glue.cu
oda_status launch_glue_hidden(oda_ctx* ctx, const float* emb, const float* terms, int n_terms,
                              const int32_t* flag, float* h, cudaStream_t stream);
oda_status launch_glue_gdn(oda_ctx* ctx, const oda_state* src, const oda_state* st, int layer,
                           const float* c, const float* v, const float* alpha, const float* beta,
                           const float* taps, const int32_t* flag, float* o, cudaStream_t s);
int glue_chunks(int D);

// backbone.cu
oda_status launch_bb_qkv(oda_ctx* ctx, const oda_bb_layer* w, const float* x, void* q, void* k_new,
                         void* v_new, cudaStream_t s);
oda_status launch_bb_attn_out(oda_ctx* ctx, const oda_bb_layer* w, const float* o, float* x, cudaStream_t s);
oda_status launch_bb_mlp(oda_ctx* ctx, const oda_bb_layer* w, float* x, void* act, cudaStream_t s);
oda_status launch_bb_begin(oda_ctx* ctx, const float* emb, float* x, cudaStream_t s);
oda_status launch_bb_pack_weight(oda_ctx* ctx, const void* src, int32_t rows, int32_t cols, void* dst,
                                 cudaStream_t s);
oda_status launch_bb_post(oda_ctx* ctx, const oda_bb_layer* w, const oda_bb_layer* next,
                          const float* o, float* x, void* act, void* q, void* k_new, void* v_new,
                          cudaStream_t s);
oda_status launch_bb_final_norm(oda_ctx* ctx, const float* gamma, const float* x, float* h, cudaStream_t s);
oda_status launch_bb_lm_head(oda_ctx* ctx, const void* embed, int32_t vocab, const float* h,
                             float* logits, int32_t* token, float* next_emb, cudaStream_t s);
oda_status launch_bb_embed(oda_ctx* ctx, const void* embed, int32_t vocab, const int32_t* token,
                           float* emb, cudaStream_t s);

// cond.cu
oda_status launch_set_condition(cudaGraphConditionalHandle h, const int32_t* any_flag,
                                bool overlap, cudaStream_t stream);

}  // namespace oda
