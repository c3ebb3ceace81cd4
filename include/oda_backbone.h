/*
 * oda_backbone.h - synthetic frozen backbone around the restricted attention layers: the
 * projections of a Qwen3-shaped decoder layer with (random) bf16 weights, and the LM head.
 *
 * Not part of the method itself: the method notes ("On-Demand Attention：让语言模型按需读取完整
 * 历史") keep the pretrained backbone frozen and change only which positions each attention layer
 * reads [notes §2.1]; their throughput figures time the whole decode step - every layer, the
 * recall head, the conditional full pass, the commit and the LM head [notes §3.3], with the
 * output distribution computed once from the committed hidden state [notes §2.3, eq. p_t].
 * These calls make that whole step runnable without trained weights.  Per attention layer:
 *   oda_bb_qkv      n = RMSNorm(x) * g_attn;  [q | k | v] = W_qkv bf16(n)   (bf16 outputs)
 *   oda_attend_*    o = attention over S^L or S^F (oda.h)
 *   oda_bb_attn_out x += W_o bf16(o)
 *   oda_bb_mlp      m = RMSNorm(x) * g_mlp;  x += W_down bf16(SiLU(W_gate bf16(m)) * W_up bf16(m))
 * then oda_bb_final_norm (h = RMSNorm(x) * g_final: the head's "last-layer normalised hidden")
 * and, after the commit, oda_bb_lm_head (logits = E bf16(h_t), greedy token, next embedding).
 * RMSNorm eps = 1e-6; no positional rotation and no per-head q/k norm.  Hidden width D =
 * Hq * 128 of the context; x, o, h fp32 [B][D]; batch <= 8.  Weight matrices are bf16 [out][in]
 * in the packed layout written by oda_bb_pack_weight (below), 16-byte aligned; D, F multiples
 * of 512; N (rows) multiples of 16.  Same
 * conventions as oda.h (device pointers, asynchronous on `stream`, no allocation, graph
 * capturable).  When the context has overlap_layers = 1 these launches overlap the previous
 * kernel of the stream (they only read weights before it finishes).
 */
#ifndef ODA_BACKBONE_H
#define ODA_BACKBONE_H

#include "oda.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  const float* attn_norm;   /* g_attn [D] fp32                                           */
  const void* w_qkv;        /* bf16 [(Hq + 2 Hkv) * 128][D]: q rows, then k, then v       */
  const void* w_o;          /* bf16 [D][Hq * 128]                                        */
  const float* mlp_norm;    /* g_mlp [D] fp32                                            */
  const void* w_gate;       /* bf16 [F][D]                                               */
  const void* w_up;         /* bf16 [F][D]                                               */
  const void* w_down;       /* bf16 [D][F]                                               */
  int32_t ffn;              /* F                                                         */
} oda_bb_layer;

/* Packed weight layout.  A matrix W [rows][cols] (bf16; rows a multiple of 16, cols of 512) is
 * stored as blocks of 16 rows x 512 columns, 8192 elements each, block (i, c) (rows 16i..16i+15,
 * columns 512c..512c+511) at element offset (i * cols / 512 + c) * 8192.  Inside a block, row r
 * (0..15) takes 512 elements at offset r * 512, made of 64 chunks of 8 consecutive columns;
 * chunk j (columns 512c + 8j .. 8j + 7) sits at slot j XOR (r mod 8).  So W[n][k] is element
 *   ((n / 16) * (cols / 512) + k / 512) * 8192 + (n % 16) * 512 + (((k % 512) / 8) ^ (n % 8)) * 8 + k % 8.
 * The projections stream a tile's K range as a few contiguous copies, and the swizzle keeps the
 * shared-memory reads of 8 rows at one column conflict-free.  Same size as the row-major matrix.
 *
 * dst = src (row-major [rows][cols] bf16) in the packed layout.  src and dst device pointers,
 * 16-byte aligned, not overlapping; asynchronous on `stream`.  ODA_ERR_INVALID_ARG for a NULL,
 * misaligned or shared pointer or a shape outside the rule above. */
oda_status oda_bb_pack_weight(oda_ctx* ctx, const void* src, int32_t rows, int32_t cols, void* dst,
                              cudaStream_t stream);

/* x <- emb (the residual stream of a pass starts from E(x_t)); fp32 [B][D]. */
oda_status oda_bb_begin(oda_ctx* ctx, const float* emb, float* x, cudaStream_t stream);

/* q [B][Hq][128], k_new, v_new [B][Hkv][128] (bf16) from the residual x (fp32 [B][D]). */
oda_status oda_bb_qkv(oda_ctx* ctx, const oda_bb_layer* layer, const float* x, void* q,
                      void* k_new, void* v_new, cudaStream_t stream);

/* x += W_o bf16(o), o = the layer's attention output fp32 [B][Hq*128]. */
oda_status oda_bb_attn_out(oda_ctx* ctx, const oda_bb_layer* layer, const float* o, float* x,
                           cudaStream_t stream);

/* The gated MLP with its input norm, in place on x; act: caller workspace, bf16 [B][F]
 * (holds the activation SiLU(gate) * up between the two launches). */
oda_status oda_bb_mlp(oda_ctx* ctx, const oda_bb_layer* layer, float* x, void* act,
                      cudaStream_t stream);

/* Everything between the attention of `layer` and the attention of `next`, in one launch:
 * oda_bb_attn_out(layer, o, x), oda_bb_mlp(layer, x, act) and, when next != NULL,
 * oda_bb_qkv(next, x, q, k_new, v_new), with the same arithmetic and outputs as those three
 * calls made in that order.  A cooperative launch of one CTA per SM whose phases are separated
 * by grid barriers (bounded waits: a barrier that does not complete within 2 s sets
 * ODA_DEVERR_WAIT_TIMEOUT in the context's device error word and the kernel runs on, so the
 * outputs are then undefined).  Launches of this call on one context must be serialised (they
 * share the barrier counters in the context), which holds for calls on one stream.  Errors:
 * ODA_ERR_INVALID_ARG for a NULL or misaligned pointer; ODA_ERR_UNSUPPORTED for shapes the
 * projections reject or a device without cooperative launch. */
oda_status oda_bb_post_attention(oda_ctx* ctx, const oda_bb_layer* layer, const oda_bb_layer* next,
                                 const float* o, float* x, void* act, void* q, void* k_new,
                                 void* v_new, cudaStream_t stream);

/* h = RMSNorm(x) * gamma (fp32 [B][D]). */
oda_status oda_bb_final_norm(oda_ctx* ctx, const float* gamma, const float* x, float* h,
                             cudaStream_t stream);

/* LM head on the committed hidden h (fp32 [B][D]) with the tied embedding table embed (bf16
 * [vocab][D] packed, vocab a multiple of 16): logits fp32 [B][vocab] = embed bf16(h); token[b] = the
 * smallest index of the largest logit; next_emb fp32 [B][D] = embed[token[b]]. */
oda_status oda_bb_lm_head(oda_ctx* ctx, const void* embed, int32_t vocab, const float* h,
                          float* logits, int32_t* token, float* next_emb, cudaStream_t stream);

/* emb[b] = embed[token[b]] as fp32, embed packed (a token outside [0, vocab) is taken as 0 and
 * written back to token[b]). */
oda_status oda_bb_embed(oda_ctx* ctx, const void* embed, int32_t vocab, int32_t* token,
                        float* emb, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ODA_BACKBONE_H */
