// Transactional commit of the chosen branch, and snapshot / restore of recurrent state.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.3: the current K,V
// of every layer are staged and only the chosen branch's update is written to the full cache
// (and with it to the local view, which here is an index set over the same cache); the
// committed hidden state comes from the same branch (eq. h_t = h^{b_t}_t, C_t = C_{t-1} ||
// dC^{b_t}_t).  Hybrid backbones snapshot conv and recurrent state before the local pass and
// restore the pre-step state before the full retry.
//
// Pure data movement: 16-byte copies, bit-exact.  The commit grid is (layers x sequences);
// the last CTA of each sequence (completion counter, no waiting) takes the hidden state and
// advances the position, after every layer of that sequence has read it.
#include "internal.h"

namespace oda {
namespace {

constexpr int kPageTok = 16;

struct CommitParams {
  void* k[ODA_MAX_LAYERS];
  void* v[ODA_MAX_LAYERS];
  int64_t n_pages[ODA_MAX_LAYERS];
  const int32_t* page_table;
  int32_t* pos;
  const int32_t* flag;
  const uint4* ks[2];     // staging [L][B][Hkv][128] bf16 as 16-byte words; [0] local, [1] full
  const uint4* vs[2];
  const float4* h[2];
  float4* h_prev;
  int32_t* cnt;           // [B]
  int32_t* err;
  int L, B, Hkv, max_pages, D4;
};

__global__ void __launch_bounds__(256) commit_kernel(const CommitParams p) {
  const int l = blockIdx.x, b = blockIdx.y;
  const int t = p.pos[b];
  const int br = p.flag[b] != 0 ? 1 : 0;
  __shared__ int s_last;
  const bool pos_ok = t >= 1 && (int64_t)t <= (int64_t)p.max_pages * kPageTok;
  if (pos_ok) {
    const int lp = (t - 1) / kPageTok, slot = (t - 1) % kPageTok;
    const int phys = p.page_table[(size_t)b * p.max_pages + lp];
    if (phys >= 0 && (int64_t)phys < p.n_pages[l]) {
      const int words = p.Hkv * 16;  // 16-byte words per token of one layer (K or V)
      const size_t src0 = ((size_t)l * p.B + b) * words;
      for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) {
        const int which = i >= words;     // 0: K, 1: V
        const int w = i - which * words;
        const int h = w >> 4, c = w & 15;
        const uint4 val = which ? p.vs[br][src0 + w] : p.ks[br][src0 + w];
        uint4* pool = reinterpret_cast<uint4*>(which ? p.v[l] : p.k[l]);
        pool[(((size_t)phys * p.Hkv + h) * kPageTok + slot) * 16 + c] = val;
      }
    } else if (threadIdx.x == 0) {
      atomicOr(p.err, ODA_DEVERR_PAGE_RANGE);
    }
  } else if (threadIdx.x == 0 && l == 0) {
    atomicOr(p.err, ODA_DEVERR_POS_RANGE);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&p.cnt[b], 1) == p.L - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (pos_ok) {
    for (int i = threadIdx.x; i < p.D4; i += blockDim.x) p.h_prev[(size_t)b * p.D4 + i] = p.h[br][(size_t)b * p.D4 + i];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (pos_ok) p.pos[b] = t + 1;
    p.cnt[b] = 0;
  }
}

// dst[b] <- src[b] for every sequence (flag == nullptr) or the flagged ones; blockIdx.y = b.
__global__ void state_copy_kernel(const float4* src, float4* dst, size_t per_seq4,
                                  const int32_t* flag) {
  const int b = blockIdx.y;
  if (flag && flag[b] == 0) return;
  const float4* s = src + (size_t)b * per_seq4;
  float4* d = dst + (size_t)b * per_seq4;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_seq4;
       i += (size_t)gridDim.x * blockDim.x)
    d[i] = s[i];
}

}  // namespace

oda_status launch_commit(oda_ctx* ctx, const oda_kv_layer* layers, int32_t n_layers,
                         const int32_t* page_table, int32_t* pos, const int32_t* flag,
                         const void* ksl, const void* vsl, const void* ksf, const void* vsf,
                         const float* h_local, const float* h_full, float* h_prev,
                         cudaStream_t stream) {
  const oda_config& cf = ctx->cfg;
  if (!layers || n_layers < 1 || n_layers > ODA_MAX_LAYERS)
    return set_error(ODA_ERR_INVALID_ARG, "commit: n_layers must be 1..%d", ODA_MAX_LAYERS);
  if (!page_table || !pos || !flag || !ksl || !vsl || !ksf || !vsf || !h_local || !h_full || !h_prev)
    return set_error(ODA_ERR_INVALID_ARG, "commit: null pointer argument");
  const void* al[] = {ksl, vsl, ksf, vsf, h_local, h_full, h_prev};
  for (const void* q : al)
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return set_error(ODA_ERR_INVALID_ARG, "commit: staging and hidden buffers must be 16-byte aligned");
  CommitParams p;
  for (int l = 0; l < n_layers; ++l) {
    if (!layers[l].k || !layers[l].v || layers[l].n_pages <= 0 ||
        ((reinterpret_cast<uintptr_t>(layers[l].k) | reinterpret_cast<uintptr_t>(layers[l].v)) & 15))
      return set_error(ODA_ERR_INVALID_ARG, "commit: bad KV pool of layer %d", l);
    p.k[l] = layers[l].k;
    p.v[l] = layers[l].v;
    p.n_pages[l] = layers[l].n_pages;
  }
  p.page_table = page_table;
  p.pos = pos;
  p.flag = flag;
  p.ks[0] = static_cast<const uint4*>(ksl);
  p.vs[0] = static_cast<const uint4*>(vsl);
  p.ks[1] = static_cast<const uint4*>(ksf);
  p.vs[1] = static_cast<const uint4*>(vsf);
  p.h[0] = reinterpret_cast<const float4*>(h_local);
  p.h[1] = reinterpret_cast<const float4*>(h_full);
  p.h_prev = reinterpret_cast<float4*>(h_prev);
  p.cnt = ctx->glue_cnt + cf.batch;  // commit's own counters
  p.err = ctx->err;
  p.L = n_layers;
  p.B = cf.batch;
  p.Hkv = cf.n_kv_heads;
  p.max_pages = cf.max_pages;
  p.D4 = cf.head_in_dim / 4;
  commit_kernel<<<dim3(n_layers, cf.batch), 256, 0, stream>>>(p);
  return check_cuda(cudaGetLastError(), "commit launch");
}

oda_status launch_state_copy(const oda_state* src, const oda_state* dst, int B,
                             const int32_t* flag, cudaStream_t stream) {
  if (!src || !dst || !src->rec || !dst->rec || !src->conv || !dst->conv)
    return set_error(ODA_ERR_INVALID_ARG, "state copy: null pointer argument");
  if (src->n_layers != dst->n_layers || src->heads != dst->heads || src->dk != dst->dk ||
      src->dv != dst->dv || src->conv_taps != dst->conv_taps || src->conv_width != dst->conv_width)
    return set_error(ODA_ERR_INVALID_ARG, "state copy: shapes differ");
  if (src->n_layers < 1 || src->heads < 1 || src->dk < 1 || src->dv < 1 || src->conv_taps < 0 ||
      src->conv_width < 0)
    return set_error(ODA_ERR_INVALID_ARG, "state copy: bad shape");
  const size_t rec = (size_t)src->n_layers * src->heads * src->dk * src->dv;
  const size_t conv = (size_t)src->n_layers * src->conv_taps * src->conv_width;
  if ((rec & 3) || (conv & 3))
    return set_error(ODA_ERR_UNSUPPORTED, "state copy: per-sequence sizes must be multiples of 4 floats");
  const void* al[] = {src->rec, dst->rec, src->conv, dst->conv};
  for (const void* q : al)
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return set_error(ODA_ERR_INVALID_ARG, "state copy: buffers must be 16-byte aligned");
  const int blocks_rec = (int)std::min<size_t>(1024, (rec / 4 + 255) / 256);
  state_copy_kernel<<<dim3(blocks_rec, B), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(src->rec), reinterpret_cast<float4*>(dst->rec), rec / 4, flag);
  oda_status st = check_cuda(cudaGetLastError(), "state copy launch");
  if (st != ODA_OK || conv == 0) return st;
  const int blocks_conv = (int)std::min<size_t>(1024, (conv / 4 + 255) / 256);
  state_copy_kernel<<<dim3(blocks_conv, B), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(src->conv), reinterpret_cast<float4*>(dst->conv), conv / 4, flag);
  return check_cuda(cudaGetLastError(), "state copy launch");
}

}  // namespace oda
