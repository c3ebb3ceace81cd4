/*
 * oda_glue.h - synthetic backbone stand-in used to drive the ODA decode step end to end.
 *
 * Not part of the method: the method notes ("On-Demand Attention：让语言模型按需读取完整历史")
 * keep the pretrained backbone frozen, and no weights are available here, so these
 * kernels stand in for everything between the restricted attention layers:
 *   - the residual stream and final RMSNorm that give the "last-layer normalised hidden"
 *     the recall head reads ([notes §2.2]),
 *   - the gated-delta recurrent layers of the hybrid backbone ([notes §3.1]: 18 Gated
 *     DeltaNet layers beside 6 attention layers), whose state the commit protocol must
 *     snapshot and restore ([notes §2.3]).
 * Same conventions as oda.h (device pointers, asynchronous, no allocation).
 */
#ifndef ODA_GLUE_H
#define ODA_GLUE_H

#include "oda.h"

#ifdef __cplusplus
extern "C" {
#endif

/* x[b] = emb[b] + sum_i terms[i][b]   (fp32, terms [n_terms][B][D], D = head_in_dim)
 * h[b] = x[b] / sqrt(mean(x[b]^2) + 1e-6)
 * If flag is non-NULL only rows with flag[b] != 0 are written.  n_terms may be 0. */
oda_status oda_glue_hidden(oda_ctx* ctx, const float* emb, const float* terms, int32_t n_terms,
                           const int32_t* flag, float* h, cudaStream_t stream);

/* One gated-delta layer (index `layer` of st) for every sequence (flag NULL) or the
 * flagged ones, advancing st->rec and st->conv in place:
 *   conv <- [conv[1..3], c];  u = sum_i taps[i] * conv[i];
 *   per head h (16 x 128): k = u_h / ||u_h||, q = k,
 *   S_h <- alpha S_h (I - beta k k^T) + beta v_h k^T,  o_h = S_h q.
 * c: [B][2048]; v: [B][16][128]; alpha, beta: [B][16]; taps: [4][2048]; o: [B][2048].
 * Requires heads = 16, dk = dv = 128, conv_taps = 4, conv_width = 2048. */
oda_status oda_glue_gdn(oda_ctx* ctx, const oda_state* st, int32_t layer, const float* c,
                        const float* v, const float* alpha, const float* beta,
                        const float* taps, const int32_t* flag, float* o, cudaStream_t stream);

/* The same layer update reading the layer's state from src and writing the advanced state to
 * dst (same shapes; src == dst is oda_glue_gdn).  With two state buffers used alternately, the
 * pre-step state of a hybrid backbone stays intact in one of them while the local pass writes
 * the other: the full retry reads it directly, so neither a snapshot copy nor a restore copy is
 * needed ([notes §2.3, third paragraph]: the retry must start from the pre-step state and no
 * state may advance twice). */
oda_status oda_glue_gdn_step(oda_ctx* ctx, const oda_state* src, const oda_state* dst,
                             int32_t layer, const float* c, const float* v, const float* alpha,
                             const float* beta, const float* taps, const int32_t* flag, float* o,
                             cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ODA_GLUE_H */
