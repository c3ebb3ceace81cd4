// Transactional commit of the chosen branch, and snapshot / restore of recurrent state.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.3: the current K,V
// of every layer are staged and only the chosen branch's update is written to the full cache
// (and with it to the local view, which here is an index set over the same cache); the
// committed hidden state comes from the same branch (eq. h_t = h^{b_t}_t, C_t = C_{t-1} ||
// dC^{b_t}_t).  Hybrid backbones snapshot conv and recurrent state before the local pass and
// restore the pre-step state before the full retry.
//
// bf16 pages: pure data movement, 16-byte copies, bit-exact.  fp8 pages: each committed token
// row is quantised (e4m3 codes, one fp32 scale per row) into its page block; the same routine
// packs a whole bf16 cache into fp8 blocks.  The commit grid is (layers x sequences);
// the last CTA of each sequence (completion counter, no waiting) takes the hidden state and
// advances the position, after every layer of that sequence has read it.
#include "internal.h"
#include "ptx.cuh"

namespace oda {
namespace {

constexpr int kPageTok = 16;

// fp8 page block of one (page, KV head): K codes [16 tokens][128] with chunk k of token j at
// chunk position k ^ (j & 7); V codes transposed [128 dims][16 slots], slot s holding token
// 2*(s/4) + (s&1) + 8*((s>>1)&1); K scales fp32 [16]; V scales fp32 [16] (4224 bytes).
constexpr int kF8Block = 4224;
constexpr int kF8V = 2048;
constexpr int kF8SK = 4096;
constexpr int kF8SV = 4160;

__device__ __forceinline__ int v8_slot(int j) { return 4 * ((j & 7) >> 1) + ((j >> 3) << 1) + (j & 1); }

// Quantises one 128-value bf16 row (this lane: values 4*lane .. 4*lane + 3, given as two bf16
// pairs) to e4m3 codes with one fp32 scale: s = max|x| / 448 (1 for an all-zero row),
// code = round-to-nearest-even(x / s) with saturation at +-448; both divisions in fp32 with
// IEEE rounding.  Returns the four codes (value 4*lane + i in byte i); *scale gets s.
__device__ __forceinline__ uint32_t quantize_row_e4m3(uint32_t w01, uint32_t w23, int lane, float* scale) {
  const float x0 = bf16_lo_to_f32(w01), x1 = bf16_hi_to_f32(w01);
  const float x2 = bf16_lo_to_f32(w23), x3 = bf16_hi_to_f32(w23);
  float amax = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  *scale = s;
  const uint32_t c01 = f32x2_to_e4m3x2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
  const uint32_t c23 = f32x2_to_e4m3x2(__fdiv_rn(x2, s), __fdiv_rn(x3, s));
  return c01 | (c23 << 16);
}

// Writes a quantised token row (K if which == 0, else V) into slot j of a block.
__device__ __forceinline__ void store_row_e4m3(uint8_t* blk, int which, int j, uint32_t codes,
                                               float scale, int lane) {
  if (which == 0) {
    const int k = lane >> 2;   // 16-dim chunk of values 4*lane .. 4*lane + 3
    *reinterpret_cast<uint32_t*>(blk + 128 * j + 16 * (k ^ (j & 7)) + 4 * (lane & 3)) = codes;
    if (lane == 0) *reinterpret_cast<float*>(blk + kF8SK + 4 * j) = scale;
  } else {
    const int sl = v8_slot(j);
#pragma unroll
    for (int i = 0; i < 4; ++i) blk[kF8V + 16 * (4 * lane + i) + sl] = (uint8_t)(codes >> (8 * i));
    if (lane == 0) *reinterpret_cast<float*>(blk + kF8SV + 4 * j) = scale;
  }
}

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

template <int F>
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
      if constexpr (F == 0) {
        for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) {
          const int which = i >= words;     // 0: K, 1: V
          const int w = i - which * words;
          const int h = w >> 4, c = w & 15;
          const uint4 val = which ? p.vs[br][src0 + w] : p.ks[br][src0 + w];
          uint4* pool = reinterpret_cast<uint4*>(which ? p.v[l] : p.k[l]);
          pool[(((size_t)phys * p.Hkv + h) * kPageTok + slot) * 16 + c] = val;
        }
      } else {
        // one warp per (head, K or V) row: quantise and write into the page block
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int row = warp; row < 2 * p.Hkv; row += blockDim.x >> 5) {
          const int which = row / p.Hkv, h = row - which * p.Hkv;
          const uint2 wv = reinterpret_cast<const uint2*>(which ? p.vs[br] : p.ks[br])[(src0 + h * 16) * 2 + lane];
          float sc;
          const uint32_t codes = quantize_row_e4m3(wv.x, wv.y, lane, &sc);
          uint8_t* blk = static_cast<uint8_t*>(p.k[l]) + ((size_t)phys * p.Hkv + h) * kF8Block;
          store_row_e4m3(blk, which, slot, codes, sc, lane);
        }
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

// Packs bf16 pools [n_pages][Hkv][16][128] (K and V) into fp8 page blocks; one CTA of 8 warps
// per (page, KV head) block, one warp per token row of K or V (32 rows).
__global__ void __launch_bounds__(256) kv8_pack_kernel(const uint2* k, const uint2* v, uint8_t* dst) {
  const size_t blkid = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* blk = dst + blkid * kF8Block;
  for (int row = warp; row < 2 * kPageTok; row += 8) {
    const int which = row >> 4, j = row & 15;
    const uint2 w = (which ? v : k)[(blkid * kPageTok + j) * 32 + lane];
    float sc;
    const uint32_t codes = quantize_row_e4m3(w.x, w.y, lane, &sc);
    store_row_e4m3(blk, which, j, codes, sc, lane);
  }
}

}  // namespace

oda_status launch_kv8_pack(const oda_kv_layer* src, const oda_kv8_layer* dst, int32_t n_kv_heads,
                           cudaStream_t stream) {
  if (!src || !dst || !src->k || !src->v || !dst->kv)
    return set_error(ODA_ERR_INVALID_ARG, "kv8_pack: null pointer argument");
  if (n_kv_heads < 1 || src->n_pages < 1 || src->n_pages != dst->n_pages ||
      src->n_pages * (int64_t)n_kv_heads > INT32_MAX)
    return set_error(ODA_ERR_INVALID_ARG, "kv8_pack: page counts differ or out of range");
  if ((reinterpret_cast<uintptr_t>(src->k) | reinterpret_cast<uintptr_t>(src->v) |
       reinterpret_cast<uintptr_t>(dst->kv)) & 15)
    return set_error(ODA_ERR_INVALID_ARG, "kv8_pack: pools must be 16-byte aligned");
  const int64_t blocks = src->n_pages * n_kv_heads;
  kv8_pack_kernel<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const uint2*>(src->k),
                                                         static_cast<const uint2*>(src->v),
                                                         static_cast<uint8_t*>(dst->kv));
  return check_cuda(cudaGetLastError(), "kv8_pack launch");
}

oda_status launch_commit(oda_ctx* ctx, const KvPool* layers, int32_t n_layers,
                         const int32_t* page_table, int32_t* pos, const int32_t* flag,
                         const void* ksl, const void* vsl, const void* ksf, const void* vsf,
                         const float* h_local, const float* h_full, float* h_prev,
                         cudaStream_t stream) {
  const oda_config& cf = ctx->cfg;
  if (!layers || n_layers < 1 || n_layers > ODA_MAX_LAYERS)
    return set_error(ODA_ERR_INVALID_ARG, "commit: n_layers must be 1..%d", ODA_MAX_LAYERS);
  const int F = layers[0].fmt;
  if (!page_table || !pos || !flag || !ksl || !vsl || !ksf || !vsf || !h_local || !h_full || !h_prev)
    return set_error(ODA_ERR_INVALID_ARG, "commit: null pointer argument");
  const void* al[] = {ksl, vsl, ksf, vsf, h_local, h_full, h_prev};
  for (const void* q : al)
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return set_error(ODA_ERR_INVALID_ARG, "commit: staging and hidden buffers must be 16-byte aligned");
  CommitParams p;
  for (int l = 0; l < n_layers; ++l) {
    if (layers[l].fmt != F || !layers[l].k || (F == 0 && !layers[l].v) || layers[l].n_pages <= 0 ||
        ((reinterpret_cast<uintptr_t>(layers[l].k) | reinterpret_cast<uintptr_t>(layers[l].v)) & 15))
      return set_error(ODA_ERR_INVALID_ARG, "commit: bad KV pool of layer %d", l);
    p.k[l] = const_cast<void*>(layers[l].k);
    p.v[l] = const_cast<void*>(layers[l].v);
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
  if (F == 0)
    commit_kernel<0><<<dim3(n_layers, cf.batch), 256, 0, stream>>>(p);
  else
    commit_kernel<1><<<dim3(n_layers, cf.batch), 256, 0, stream>>>(p);
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
