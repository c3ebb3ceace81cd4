// Synthetic backbone stand-in (not the method): residual + final RMSNorm, gated-delta layer.
//
// The method notes ("On-Demand Attention：让语言模型按需读取完整历史") keep the backbone frozen;
// without weights, the decode step is driven by seeded per-layer inputs, a residual stream
// x = E(x_t) + sum of layer outputs, and h = RMSNorm(x) (the "last-layer normalised hidden"
// of §2.2).  The hybrid workload's 18 linear-recurrent layers (§3.1: Gated DeltaNet) are
// stood in for by a 4-tap causal conv plus the gated delta rule on a 16 x 128 x 128 state.
#include "internal.h"
#include "ptx.cuh"

namespace oda {
namespace {

constexpr int kGlueChunk = 256;
constexpr float kEps = 1e-6f;

__device__ float block_sum256(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
  __syncthreads();
  return s;
}

__global__ void __launch_bounds__(kGlueChunk)
hidden_kernel(const float* emb, const float* terms, int n_terms, const int32_t* flag, float* h,
              float* xbuf, float* ssbuf, int32_t* cnt, int B, int D) {
  const int b = blockIdx.y, chunk = blockIdx.x, nch = gridDim.x;
  // launched with programmatic dependent launch: wait for the kernels that wrote the layer
  // outputs (and the flags) before reading anything, and let the recall head start early
  grid_dependency_wait();
  grid_dependents_launch();
  if (flag && flag[b] == 0) return;
  __shared__ float red[kGlueChunk / 32];
  __shared__ int s_last;
  const int d = chunk * kGlueChunk + threadIdx.x;
  float x = 0.f;
  if (d < D) {
    // four partial sums (term i goes to sum i mod 4, in increasing i); the loads of twelve
    // terms are issued before any of them is added, so they are in flight together
    const float* tp = terms + (size_t)b * D + d;
    const size_t stride = (size_t)B * D;
    float a0 = emb[(size_t)b * D + d], a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int i = 0;
    for (; i + 12 <= n_terms; i += 12) {
      float v[12];
#pragma unroll
      for (int j = 0; j < 12; ++j) v[j] = tp[(size_t)(i + j) * stride];
#pragma unroll
      for (int j = 0; j < 12; j += 4) {
        a0 += v[j];
        a1 += v[j + 1];
        a2 += v[j + 2];
        a3 += v[j + 3];
      }
    }
    for (; i + 4 <= n_terms; i += 4) {
      a0 += tp[(size_t)i * stride];
      a1 += tp[(size_t)(i + 1) * stride];
      a2 += tp[(size_t)(i + 2) * stride];
      a3 += tp[(size_t)(i + 3) * stride];
    }
    for (; i < n_terms; ++i) a0 += tp[(size_t)i * stride];
    x = (a0 + a1) + (a2 + a3);
    xbuf[(size_t)b * D + d] = x;
  }
  const float ss = block_sum256(x * x, red);
  if (threadIdx.x == 0) ssbuf[(size_t)b * nch + chunk] = ss;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&cnt[b], 1) == nch - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float tot = 0.f;
  for (int c = 0; c < nch; ++c) tot += __ldcg(ssbuf + (size_t)b * nch + c);
  const float inv = rsqrtf(tot / D + kEps);
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    h[(size_t)b * D + i] = __ldcg(xbuf + (size_t)b * D + i) * inv;
  if (threadIdx.x == 0) cnt[b] = 0;
}

// One (sequence, head) per CTA of 256 threads: thread t owns half of row t/2 of S_h.  The layer's
// state is read from (rec_in, conv_in) and the advanced state written to (rec_out, conv_out);
// the two may be the same buffers (in place) or different ones (the pre-step state stays).
__global__ void __launch_bounds__(256)
gdn_kernel(const float* rec_in, const float* conv_in, float* rec, float* conv, int n_layers,
           int layer, const float* c, const float* v, const float* alpha, const float* beta,
           const float* taps, const int32_t* flag, float* o) {
  constexpr int H = 16, DK = 128, W = 2048, TAPS = 4;
  const int h = blockIdx.x, b = blockIdx.y;
  if (flag && flag[b] == 0) return;
  __shared__ float k_s[DK];
  __shared__ float red[8];
  const int tid = threadIdx.x;
  const float* ci = conv_in + ((size_t)b * n_layers + layer) * TAPS * W;
  float* cv = conv + ((size_t)b * n_layers + layer) * TAPS * W;
  float u = 0.f;
  if (tid < DK) {
    const int e = h * DK + tid;
    const float c0 = ci[1 * W + e], c1 = ci[2 * W + e], c2 = ci[3 * W + e];
    const float c3 = c[(size_t)b * W + e];
    cv[0 * W + e] = c0;
    cv[1 * W + e] = c1;
    cv[2 * W + e] = c2;
    cv[3 * W + e] = c3;
    u = taps[0 * W + e] * c0 + taps[1 * W + e] * c1 + taps[2 * W + e] * c2 + taps[3 * W + e] * c3;
  }
  const float nrm2 = block_sum256(u * u, red);
  if (tid < DK) k_s[tid] = u / sqrtf(nrm2);
  __syncthreads();
  const float* Si = rec_in + (((size_t)b * n_layers + layer) * H + h) * DK * DK;
  float* S = rec + (((size_t)b * n_layers + layer) * H + h) * DK * DK;
  const int i = tid >> 1, j0 = (tid & 1) * 64;
  float4 row[16];
  float sk = 0.f;
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    row[q] = reinterpret_cast<const float4*>(Si + (size_t)i * DK + j0)[q];
    const int j = j0 + 4 * q;
    sk += row[q].x * k_s[j] + row[q].y * k_s[j + 1] + row[q].z * k_s[j + 2] + row[q].w * k_s[j + 3];
  }
  sk += __shfl_xor_sync(0xffffffffu, sk, 1);
  const float a = alpha[b * H + h], be = beta[b * H + h];
  const float vi = v[((size_t)b * H + h) * DK + i];
  // alpha S (I - beta k k^T) + beta v k^T  =  alpha S + beta (v - alpha S k) k^T
  const float coef = be * (vi - a * sk);
  float oi = 0.f;
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int j = j0 + 4 * q;
    float4 r = row[q];
    r.x = a * r.x + coef * k_s[j];
    r.y = a * r.y + coef * k_s[j + 1];
    r.z = a * r.z + coef * k_s[j + 2];
    r.w = a * r.w + coef * k_s[j + 3];
    reinterpret_cast<float4*>(S + (size_t)i * DK + j0)[q] = r;
    oi += r.x * k_s[j] + r.y * k_s[j + 1] + r.z * k_s[j + 2] + r.w * k_s[j + 3];
  }
  oi += __shfl_xor_sync(0xffffffffu, oi, 1);
  if ((tid & 1) == 0) o[(size_t)b * (H * DK) + h * DK + i] = oi;
}

}  // namespace

int glue_chunks(int D) { return (D + kGlueChunk - 1) / kGlueChunk; }

oda_status launch_glue_hidden(oda_ctx* ctx, const float* emb, const float* terms, int n_terms,
                              const int32_t* flag, float* h, cudaStream_t stream) {
  if (!emb || !h || n_terms < 0 || (n_terms > 0 && !terms))
    return set_error(ODA_ERR_INVALID_ARG, "glue_hidden: bad argument");
  const int B = ctx->cfg.batch, D = ctx->cfg.head_in_dim;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(glue_chunks(D), B);
  lc.blockDim = dim3(kGlueChunk);
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = ctx->cfg.overlap_layers ? 1 : 0;
  return check_cuda(cudaLaunchKernelEx(&lc, hidden_kernel, emb, terms, n_terms, flag, h,
                                       ctx->glue_x, ctx->glue_ss, ctx->glue_cnt, B, D),
                    "glue_hidden launch");
}

oda_status launch_glue_gdn(oda_ctx* ctx, const oda_state* src, const oda_state* st, int layer,
                           const float* c, const float* v, const float* alpha, const float* beta,
                           const float* taps, const int32_t* flag, float* o, cudaStream_t s) {
  if (!src || !st || !st->rec || !st->conv || !src->rec || !src->conv || !c || !v || !alpha ||
      !beta || !taps || !o)
    return set_error(ODA_ERR_INVALID_ARG, "glue_gdn: null pointer argument");
  if (st->heads != 16 || st->dk != 128 || st->dv != 128 || st->conv_taps != 4 ||
      st->conv_width != 2048)
    return set_error(ODA_ERR_UNSUPPORTED, "glue_gdn: needs 16 heads of 128x128 and a 4x2048 conv");
  if (src->n_layers != st->n_layers || src->heads != st->heads || src->dk != st->dk ||
      src->dv != st->dv || src->conv_taps != st->conv_taps || src->conv_width != st->conv_width)
    return set_error(ODA_ERR_INVALID_ARG, "glue_gdn: source and destination shapes differ");
  if (layer < 0 || layer >= st->n_layers)
    return set_error(ODA_ERR_INVALID_ARG, "glue_gdn: layer %d out of range", layer);
  if ((reinterpret_cast<uintptr_t>(st->rec) | reinterpret_cast<uintptr_t>(src->rec)) & 15)
    return set_error(ODA_ERR_INVALID_ARG, "glue_gdn: state must be 16-byte aligned");
  gdn_kernel<<<dim3(16, ctx->cfg.batch), 256, 0, s>>>(src->rec, src->conv, st->rec, st->conv,
                                                       st->n_layers, layer, c, v, alpha, beta, taps,
                                                       flag, o);
  return check_cuda(cudaGetLastError(), "glue_gdn launch");
}

}  // namespace oda
