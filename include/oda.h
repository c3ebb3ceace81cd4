/*
 * oda.h - C ABI of the On-Demand Attention (ODA) decode hot path for NVIDIA B200 (sm_100a).
 *
 * Method (web page "On-Demand Attention：让语言模型按需读取完整历史", the method notes,
 * cited below as [notes §n]): every decode step first runs a local pass whose restricted
 * attention layers read the index set S^L_t = {1..min(s,t)} U {max(1,t-w+1)..t} (s = 4 sinks,
 * w = 2048 window including the current token) of a fully retained KV cache; a recall head
 * R(h_{t-1}, E(x_t), h^L_t) scores the step; where the score exceeds theta (0) or is not
 * finite, the full pass is recomputed from the same pre-step state over S^F_t = {1..t};
 * finally only the chosen branch's hidden state and current K,V are committed.
 *
 * Conventions for every entry point
 *   - Device pointers unless stated otherwise; nothing is retained after the call returns.
 *     The caller owns all tensors and streams; the context owns only its scratch.
 *   - Every call is asynchronous on the given stream, allocates nothing after oda_create,
 *     never synchronises with the host (except oda_get_error / oda_create / oda_destroy) and
 *     can be captured in a CUDA graph.  Calls on one context must be ordered on one stream
 *     (they share scratch).
 *   - Argument and shape errors return synchronously (ODA_ERR_INVALID_ARG /
 *     ODA_ERR_UNSUPPORTED) and launch nothing.  A failed launch returns ODA_ERR_CUDA.
 *     Data-dependent violations found on the device (page-table entry outside the pool,
 *     position beyond capacity, a bounded wait that gave up) set bits in the context's sticky
 *     device error word, skip the offending access, and are read with oda_get_error.
 *     Kernels never trap.  oda_last_error() gives a message for the last non-OK status of
 *     the calling thread.
 *   - Positions: pos[b] = t, the 1-based position of the token being decoded.  The cache of
 *     sequence b holds positions 1..t-1 at token indices 0..t-2; position t (the current
 *     token) is passed as staged k_new / v_new and is never read from the cache.
 *
 * Layouts
 *   KV pool of one layer (K and V separately): bf16 [n_pages][Hkv][16][128]; each
 *   (page, kv head) block is a contiguous 4 KiB.  page_table: int32 [B][max_pages],
 *   logical page p of sequence b -> physical page page_table[b*max_pages + p]; the table is
 *   shared by all layers.  q: bf16 [B][Hq][128].  k_new, v_new: bf16 [B][Hkv][128].
 *   out: fp32 [B][Hq][128].  Query head h reads KV head h / (Hq/Hkv).
 */
#ifndef ODA_H
#define ODA_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ODA_VERSION_MAJOR 0
#define ODA_VERSION_MINOR 1

typedef enum {
  ODA_OK = 0,
  ODA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or alignment                   */
  ODA_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement               */
  ODA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed                   */
  ODA_ERR_DEVICE = 4,        /* oda_get_error found the device error word non-zero     */
  ODA_ERR_STATE = 5          /* call out of order (e.g. oda_cond_end without begin)    */
} oda_status;

/* Bits of the sticky device error word. */
#define ODA_DEVERR_PAGE_RANGE   0x1  /* page-table entry outside [0, n_pages): access skipped  */
#define ODA_DEVERR_POS_RANGE    0x2  /* pos < 1 or t-1 beyond the table's capacity            */
#define ODA_DEVERR_WAIT_TIMEOUT 0x4  /* a bounded wait on a copy barrier gave up              */

#define ODA_MAX_BATCH 256
#define ODA_MAX_LAYERS 64

typedef struct oda_ctx oda_ctx;

typedef struct {
  int32_t batch;        /* B, 1..ODA_MAX_BATCH                                        */
  int32_t n_q_heads;    /* Hq                                                          */
  int32_t n_kv_heads;   /* Hkv; Hq % Hkv == 0 and g = Hq / Hkv in 1..8                  */
  int32_t head_dim;     /* d_k; must be 128                                            */
  int32_t page_size;    /* tokens per page; must be 16                                 */
  int32_t max_pages;    /* pages per sequence = row length of the page table           */
  int32_t sinks;        /* s (the notes use 4), 0..16                                   */
  int32_t window;       /* w (the notes use 2048), >= 1, includes the current token    */
  int32_t head_in_dim;  /* D: width of each recall-head input; multiple of 512, <= 8192 */
  float theta;          /* routing threshold (the notes use 0)                          */
  int32_t overlap_layers; /* 1: two consecutive attention calls of this context overlap
                           * (programmatic dependent launch): the later call prefetches its
                           * pages while the earlier one finishes.  The caller then must not
                           * write pos, flag, the page table or the KV pools on the stream
                           * between two consecutive attention calls.  The hidden-state glue
                           * and the conditional's set-condition kernel are then launched the
                           * same way; they read nothing before the previous kernel completes.
                           * 0: every call starts after all prior work on the stream.      */
  int32_t deterministic;  /* 1: the full-set attention gives the pages of each (sequence, KV
                           * head) to its CTAs in a fixed pattern, so every launch rounds the
                           * same way (bit-identical replays).  0: pages are claimed at run time
                           * by whichever CTA is free (faster on an unevenly loaded GPU; the
                           * fp32 rounding of the output may differ from run to run within the
                           * attention tolerance).                                          */
} oda_config;

typedef struct {
  void* k;              /* bf16 [n_pages][Hkv][16][128], 16-byte aligned               */
  void* v;              /* bf16 [n_pages][Hkv][16][128], 16-byte aligned               */
  int64_t n_pages;      /* pages in this layer's pool (bounds every page-table entry)   */
} oda_kv_layer;

/* fp8 (OCP E4M3FN) KV pages.  The method notes suggest (summary and limits, section 4; the
 * review page's section 六 likewise) combining the access policy with a quantised KV cache
 * without fixing a format; this library's format keeps one fp32 scale per (token, KV head) row
 * of 128 values: s = max|x| / 448 (1 for an all-zero row; NaN values ignored), code =
 * round-to-nearest-even(x / s) saturating at +-448, both divisions in fp32 with IEEE rounding;
 * cached value = s * e4m3(code).  One layer's pool is an array of page blocks
 * [n_pages][Hkv][ODA_KV8_BLOCK_BYTES bytes]; the block of one (page, KV head) is
 *   bytes [0, 2048)     K codes: token j (0..15) of the page at 128*j; the 16-value chunk k
 *                       (0..7) of the token's 128 values is stored at chunk position k ^ (j & 7)
 *                       within its row (an XOR swizzle for conflict-free shared-memory reads);
 *   bytes [2048, 4096)  V codes transposed: dimension d (0..127) at 2048 + 16*d, 16 slots per
 *                       dimension, slot s holding token 2*(s/4) + (s%2) + 8*((s/2)%2)
 *                       (slots 4c..4c+3 hold tokens 2c, 2c+1, 2c+8, 2c+9);
 *   bytes [4096, 4160)  K scales, fp32 [16], token order;
 *   bytes [4160, 4224)  V scales, fp32 [16], token order.
 * A block holds 16 tokens in 4224 bytes: 264 bytes per token and KV head, 51.6% of bf16's 512. */
#define ODA_KV8_BLOCK_BYTES 4224

typedef struct {
  void* kv;             /* page blocks [n_pages][Hkv][4224 bytes], 16-byte aligned          */
  int64_t n_pages;      /* pages in this layer's pool (bounds every page-table entry)       */
} oda_kv8_layer;

/* Recall-head parameters, fp32, row-major [out][in] matrices.  Towers i = 0,1,2 read
 * h_{t-1}, E(x_t), h^L_t.  D = head_in_dim, T = 1024 (tower width), F = 2048 (FFN width). */
typedef struct {
  const float* tower_norm[3];  /* [D]        RMSNorm weight of each input              */
  const float* tower_w[3];     /* [T][D]                                                */
  const float* tower_b[3];     /* [T]                                                   */
  const float* fuse_w;         /* [T][9T]    interaction projection                     */
  const float* fuse_b;         /* [T]                                                   */
  const float* ffn_norm[2];    /* [T]                                                   */
  const float* ffn_gate[2];    /* [F][T]                                                */
  const float* ffn_up[2];      /* [F][T]                                                */
  const float* ffn_down[2];    /* [T][F]                                                */
  const float* out_norm;       /* [T]                                                   */
  const float* out_w;          /* [T]                                                   */
  const float* out_b;          /* [1]                                                   */
} oda_head_weights;

/* Gradient buffers of the recall head: the same tensors and shapes as oda_head_weights,
 * written (overwritten) by oda_recall_grad. */
typedef struct {
  float* tower_norm[3];
  float* tower_w[3];
  float* tower_b[3];
  float* fuse_w;
  float* fuse_b;
  float* ffn_norm[2];
  float* ffn_gate[2];
  float* ffn_up[2];
  float* ffn_down[2];
  float* out_norm;
  float* out_w;
  float* out_b;
} oda_head_grads;

/* Recurrent and conv state of the linear-recurrent layers of a hybrid backbone, fp32.
 * rec: [B][n_layers][heads][dv][dk]; conv: [B][n_layers][conv_taps][conv_width]. */
typedef struct {
  float* rec;
  float* conv;
  int32_t n_layers, heads, dk, dv, conv_taps, conv_width;
} oda_state;

/* ---------------------------------------------------------------- context ---------- */

/* Validates the configuration and allocates the context's scratch on the current device
 * (split-KV partials, completion counters, recall-head intermediates, the device error
 * word).  May synchronise.  *out is NULL on failure. */
oda_status oda_create(const oda_config* cfg, oda_ctx** out);

/* Frees the scratch (synchronises the device).  NULL is accepted. */
oda_status oda_destroy(oda_ctx* ctx);

/* ----------------------------------------------------------- attention ------------ */

/* Local-branch attention of one layer for all B sequences.  [notes §2.1, eq. o_t with
 * S_t = S^L_t, eq. S^F/S^L]: o = softmax(q K~[S^L]^T / sqrt(128)) V~[S^L], where K~, V~ are
 * the cached positions 1..t-1 followed by the staged current (k_new, v_new) at position t.
 * Writes out[b][h][:] for every b and h; never writes the cache. */
oda_status oda_attend_local(oda_ctx* ctx, const oda_kv_layer* layer, const int32_t* page_table,
                            const int32_t* pos, const void* q, const void* k_new,
                            const void* v_new, float* out, cudaStream_t stream);

/* Full-branch attention of one layer, gated per sequence by the device flag.
 * [notes §2.3]: the full pass runs only where the recall head fired; here over
 * S^F_t = {1..t} [notes §2.1].  Sequences with flag[b] == 0 do no work and their rows of out
 * are left untouched.  The host never reads the flags. */
oda_status oda_attend_full_if(oda_ctx* ctx, const oda_kv_layer* layer, const int32_t* page_table,
                              const int32_t* pos, const int32_t* flag, const void* q,
                              const void* k_new, const void* v_new, float* out,
                              cudaStream_t stream);

/* Allocation-free variant of oda_attend_full_if (the method notes have no counterpart: this
 * is a deployment convenience).  Same computation, arguments and layouts, without a context:
 * its scratch (split partials and completion counters) lives in a static device array of
 * 4 MiB that every GPU loading the library holds until exit, so the call allocates nothing.
 * It is meant for callers that cannot allocate device memory: code running inside a host
 * framework that only lends it buffers, or a latency-critical loop where cudaMalloc's
 * implicit device synchronisation is not acceptable.
 *   - cfg: the shape, checked by the same rules as oda_create except that head_in_dim, theta
 *     and overlap_layers are ignored.
 *   - It launches the same persistent grid as a context on the same device would (two CTAs
 *     per SM where the group's shared memory allows it, else one), so with
 *     cfg->deterministic = 1 its outputs are bit-identical to oda_attend_full_if's; with 0
 *     both round within the attention tolerance of each other.
 *   - device_error: optional device int32 that receives sticky ODA_DEVERR_* bits (OR-ed in,
 *     never cleared by the call); NULL keeps them in the static scratch, unread.
 *   - Scratch needed, in bytes, with P = B*Hkv, S = grid + P (grid as above, 148 or 296 CTAs
 *     on a B200) and g = Hq/Hkv:  roundup256(8*P + 4) + roundup256(8*g*S) + 512*g*S.  A shape
 *     needing more than the array holds is refused with ODA_ERR_UNSUPPORTED, launching nothing.
 *   - The first call on a device (and the first for each group size g) looks up the array's
 *     device address and sets the kernel's shared-memory limit (with that device current);
 *     make that first call before any stream capture.  Each call clears the counters it needs
 *     with cudaMemsetAsync on `stream`.
 *   - All calls share the one array: calls that may overlap on the GPU (other streams, other
 *     host threads) race and must be serialised by the caller. */
oda_status oda_attend_full_if_noalloc(const oda_config* cfg, const oda_kv_layer* layer,
                                      const int32_t* page_table, const int32_t* pos,
                                      const int32_t* flag, const void* q, const void* k_new,
                                      const void* v_new, float* out, int32_t* device_error,
                                      cudaStream_t stream);

/* The same two attention calls over an fp8 pool (format above): identical arguments and
 * semantics, with `layer` an fp8 pool.  The current token (position t) still comes from the
 * bf16 staging, exactly as computed by the branch (it is quantised only when committed).
 * Scores and outputs use the decoded cache values s * e4m3(code); arithmetic: codes and q
 * (scaled per head by a power of two) as f16 tensor-core operands with fp32 accumulation. */
oda_status oda_attend_local_fp8(oda_ctx* ctx, const oda_kv8_layer* layer,
                                const int32_t* page_table, const int32_t* pos, const void* q,
                                const void* k_new, const void* v_new, float* out,
                                cudaStream_t stream);
oda_status oda_attend_full_if_fp8(oda_ctx* ctx, const oda_kv8_layer* layer,
                                  const int32_t* page_table, const int32_t* pos,
                                  const int32_t* flag, const void* q, const void* k_new,
                                  const void* v_new, float* out, cudaStream_t stream);

/* Packs a bf16 cache layer (pools [n_pages][Hkv][16][128], as oda_kv_layer) into fp8 page
 * blocks, every slot of every page (slots not yet written are packed too; they are never
 * read).  src and dst must have the same n_pages.  Asynchronous on `stream`; no context. */
oda_status oda_kv8_pack(const oda_kv_layer* src, const oda_kv8_layer* dst, int32_t n_kv_heads,
                        cudaStream_t stream);

/* The index sets as the attention kernels visit them (same work decomposition): for each
 * sequence b (mode 0: all, S^L; mode 1: flag[b] != 0, S^F), positions[b*cap + i] receives the
 * 1-based cache positions read, in page order, followed by t (the staged token);
 * counts[b] the number written (0 for skipped sequences).  A debug and test entry point:
 * one thread per sequence.  Writes at most cap entries per sequence. */
oda_status oda_index_positions(oda_ctx* ctx, int32_t mode, const int32_t* pos, const int32_t* flag,
                               int32_t* positions, int32_t cap, int32_t* counts,
                               cudaStream_t stream);

/* ------------------------------------------------------------ recall head ---------- */

/* Recall score and gate for all B sequences.  [notes §2.2, eq. q_t]: q_t = R(h_{t-1},
 * E(x_t), h^L_t) with inputs h_prev, emb, h_loc (fp32 [B][D]); [notes §2.3]:
 * flag[b] = (score[b] > theta) || !isfinite(score[b]).  If sched is non-NULL the head still
 * runs but flag[b] = (sched[b] != 0) (hand-scheduled full calls, [notes §3.3]).
 * *any_flag = OR of flag[b] (int32, device).  Layer arrangement (the notes fix the three
 * inputs, the 1024-wide towers, the 9216-d interaction, two gated blocks of 2048 and the scalar
 * output; this library reads them as):
 *   u_i = SiLU(W_i (RMSNorm(x_i) * gamma_i) + b_i),  x = (h_prev, emb, h_loc)
 *   z   = [u_0, u_1, u_2, u_0*u_1, u_0*u_2, u_1*u_2, |u_0-u_1|, |u_0-u_2|, |u_1-u_2|]
 *   f   = W_f z + b_f + (u_0 + u_1 + u_2) / 3
 *   f  += W_d (SiLU(W_g m) * (W_u m)),  m = RMSNorm(f) * gamma_j      (two blocks)
 *   q   = w_o . (RMSNorm(f) * gamma_o) + b_o
 * All arithmetic fp32 with a fixed reduction order (deterministic).  The whole batch runs in
 * one cooperative launch (groups of up to 8 sequences on shares of the SMs) where D is a
 * multiple of 1024 and the inputs fit shared memory, else in six phase launches. */
oda_status oda_recall_score(oda_ctx* ctx, const oda_head_weights* w, const float* h_prev,
                            const float* emb, const float* h_loc, const int32_t* sched,
                            float* score, int32_t* flag, int32_t* any_flag, cudaStream_t stream);

/* Which path oda_recall_score takes for this context's batch and head_in_dim (host only, no
 * launch): *tile = sequences per tile of the single cooperative launch (4 or 8), *groups = its
 * sequence groups, *ring = its weight-ring depth in 32 KiB stages; all three 0 where the six
 * phase launches run.  ODA_ERR_INVALID_ARG on a NULL argument. */
oda_status oda_recall_plan(oda_ctx* ctx, int32_t* tile, int32_t* groups, int32_t* ring);

/* Training-side arithmetic of the recall head (the head is the only trained part).
 * [notes §2.1, eq. g_t]: gain g = ln p_full - ln p_local (nats), where p_full and p_local are
 * the probabilities of the next token under the full and the local pass; [notes §2.2, eqs.
 * d_t, y_t]: d = g - lambda, label y = sign(d) ln(1 + |d|); [notes §2.2, eq. L(psi)]: loss =
 * mean over the valid sequences (valid[b] != 0: reference label valid and the two access sets
 * different) of Huber with threshold 1 of q - y, 0 when none is valid.  Computes, on `stream`:
 * q [B] (the head's scores, as oda_recall_score computes them up to rounding order), y [B]
 * (0 where not valid), loss [1], and the gradient of the loss with respect to every head
 * parameter into `grad` (summed over the batch; every buffer overwritten).  The absolute
 * differences of the interaction take sign(0) = 0.  h_prev, emb, h_loc: fp32 [B][D] device.
 * All arithmetic fp32 with fixed reduction orders (deterministic).
 * Limits: 1 <= batch <= 16; head_in_dim a multiple of 1024 in 1024..8192.  Matrices, their
 * gradients, the inputs and the workspace must be 16-byte aligned.  `workspace` is device
 * memory of at least oda_recall_grad_workspace_bytes(batch, head_in_dim) bytes, owned by the
 * caller, not used across calls.  No context is needed (the call allocates nothing). */
size_t oda_recall_grad_workspace_bytes(int32_t batch, int32_t head_in_dim);
oda_status oda_recall_grad(const oda_head_weights* w, const oda_head_grads* grad, int32_t batch,
                           int32_t head_in_dim, const float* h_prev, const float* emb,
                           const float* h_loc, const float* p_full, const float* p_local,
                           const int32_t* valid, float lambda, float* loss, float* q, float* y,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------- commit -------------- */

/* Transactional commit.  [notes §2.3, eq. h_t = h^{b_t}_t, C_t = C_{t-1} || dC^{b_t}_t]:
 * for each sequence b with branch = flag[b] ? full : local and t = pos[b]:
 *   every layer l: K/V pool slot of position t (page_table[b][(t-1)/16], slot (t-1)%16)
 *                  <- k_stage_<branch>[l][b], v_stage_<branch>[l][b]  (bit-exact copy);
 *   h_prev[b] <- h_<branch>[b] (fp32 [B][D]);  pos[b] <- t + 1.
 * Staging layouts: bf16 [n_layers][B][Hkv][128].  layers: host array of n_layers entries.
 * The only writer of the cache; writes exactly one position per sequence per layer. */
oda_status oda_commit(oda_ctx* ctx, const oda_kv_layer* layers, int32_t n_layers,
                      const int32_t* page_table, int32_t* pos, const int32_t* flag,
                      const void* k_stage_local, const void* v_stage_local,
                      const void* k_stage_full, const void* v_stage_full,
                      const float* h_local, const float* h_full, float* h_prev,
                      cudaStream_t stream);

/* oda_commit for an fp8 cache: the chosen branch's staged K,V (bf16) of every layer are
 * quantised (the format above: one scale per (token, KV head) row) into the page slot of
 * position t; h_prev and pos as oda_commit.  The codes and scales written are a deterministic
 * function of the staged bf16 values. */
oda_status oda_commit_fp8(oda_ctx* ctx, const oda_kv8_layer* layers, int32_t n_layers,
                          const int32_t* page_table, int32_t* pos, const int32_t* flag,
                          const void* k_stage_local, const void* v_stage_local,
                          const void* k_stage_full, const void* v_stage_full,
                          const float* h_local, const float* h_full, float* h_prev,
                          cudaStream_t stream);

/* ----------------------------------------------------- snapshot / restore ---------- */

/* [notes §2.3, third paragraph]: hybrid backbones save the conv and recurrent state before
 * the local pass and restore the pre-step state before the full retry, so no state is
 * advanced twice.  oda_snapshot copies live -> snap for all B sequences; oda_restore copies
 * snap -> live for sequences with flag[b] != 0 only.  Bit-exact copies; both structs (host
 * pointers) must describe the same shape. */
oda_status oda_snapshot(oda_ctx* ctx, const oda_state* live, const oda_state* snap,
                        cudaStream_t stream);
oda_status oda_restore(oda_ctx* ctx, const int32_t* flag, const oda_state* snap,
                       const oda_state* live, cudaStream_t stream);

/* --------------------------------------------------- conditional retry ------------- */

/* GPU-side conditional execution of the full retry ([notes §3.3]: conditional execution
 * and CUDA Graphs keep the branch decision on the device).  If `stream` is being captured,
 * oda_cond_begin appends a kernel that sets an IF condition from *any_flag (device int32)
 * and an IF conditional node, and starts capturing the node's body on an internal stream
 * returned in *body_stream; work issued there until oda_cond_end runs only when
 * *any_flag != 0 at replay.  If `stream` is not capturing, *body_stream = stream and the
 * retry's kernels read the per-sequence flags themselves. */
oda_status oda_cond_begin(oda_ctx* ctx, cudaStream_t stream, const int32_t* any_flag,
                          cudaStream_t* body_stream);
oda_status oda_cond_end(oda_ctx* ctx, cudaStream_t stream);

/* --------------------------------------------------------- CUDA graphs ------------- */

typedef struct oda_graph oda_graph;
/* Begin capturing `stream` (relaxed mode).  Work enqueued until oda_graph_end is recorded. */
oda_status oda_graph_begin(cudaStream_t stream);
/* End the capture and instantiate it; *out owns the executable graph. */
oda_status oda_graph_end(cudaStream_t stream, oda_graph** out);
oda_status oda_graph_launch(oda_graph* g, cudaStream_t stream);
oda_status oda_graph_destroy(oda_graph* g);

/* ------------------------------------------------------------- errors -------------- */

/* Diagnostic of the bounded waits (no counterpart in the method notes): runs, on `stream`,
 * one wait that can never complete, through the same device helpers the kernels use, with a
 * limit of limit_ns (1 us .. 1 s).  which = 0: an mbarrier wait with no arrival (the page and
 * weight copy rings); which = 1: the grid-wide phase barrier of the fused recall head, with a
 * target one CTA above the grid.  The wait gives up after the limit, sets
 * ODA_DEVERR_WAIT_TIMEOUT in the context's error word and returns; the context stays usable
 * (clear the word with oda_clear_error).  No fault, trap or endless loop is involved. */
oda_status oda_probe_wait(oda_ctx* ctx, int32_t which, int64_t limit_ns, cudaStream_t stream);

/* Waits for all work on the device, then reads (and keeps) the sticky device error word into
 * *device_error (host int32).  Returns ODA_ERR_DEVICE if it is non-zero. */
oda_status oda_get_error(oda_ctx* ctx, int32_t* device_error);
oda_status oda_clear_error(oda_ctx* ctx, cudaStream_t stream);
const char* oda_status_string(oda_status s);
const char* oda_last_error(void);
int32_t oda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ODA_H */
