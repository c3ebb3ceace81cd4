// Synthetic frozen backbone around the restricted attention layers: the projections of a
// Qwen3-shaped decoder layer with random bf16 weights, and the LM head.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.1 keeps the
// pretrained backbone frozen and changes only which positions attention reads; §3.3 times the
// whole decode step (all layers, the recall head, the conditional full pass, the commit and the
// LM head), and §2.3 (eq. h_t, p_t) computes the output distribution once, from the committed
// hidden state.  No weights exist here; these kernels stand in for the backbone:
//   n = RMSNorm(x) * g_attn;  [q | k | v] = W_qkv bf16(n)           (bf16 out, to the staging)
//   x += W_o bf16(o)                                                  (o: attention output)
//   m = RMSNorm(x) * g_mlp;   a = bf16(SiLU(W_gate bf16(m)) * W_up bf16(m));  x += W_down a
//   h = RMSNorm(x) * g_final;  logits = E bf16(h_t);  token = argmax;  E(x_{t+1}) = E[token]
//
// Every projection is a weight-streaming GEMV (batch <= 8, 2 flops per 2-byte weight and
// sequence): HBM-bound.  The tensor cores take the products anyway (mma.sync m16n8k16 bf16 ->
// fp32 with weights as M and the batch as N), so the SMs only move bytes: each lane loads 16
// bytes of a weight row straight from global memory into an A fragment register group, with the
// K dimension permuted so that one 16-byte load feeds two MMA k-steps; the bf16 input vectors sit
// in shared memory in the same permuted order.  A CTA owns 16-row output tiles (its 8 warps split
// K and reduce in shared memory in a fixed order), so every output element has one writer and
// the epilogue (bf16 rounding into the staging, residual add, SiLU(gate) * up, logits) runs in
// the same kernel.  Launches overlap the previous kernel (programmatic dependent launch): a CTA
// pulls its weight tiles toward L2 before waiting for the inputs.
#include <algorithm>
#include <cmath>
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace oda {
namespace {

constexpr int kBW = 8;                 // warps per CTA (they split K)
constexpr int kBThreads = kBW * 32;
constexpr int kTile = 16;              // output rows per tile
constexpr int kMaxB = 8;               // sequences: the MMA's N
constexpr int kPad = 32;               // bf16 padding of an input row in shared memory
constexpr float kEps = 1e-6f;

enum Epi { kEpiQKV = 0, kEpiResid = 1, kEpiGateUp = 2, kEpiLogits = 3 };
enum In { kInNorm = 0, kInF32 = 1, kInBf16 = 2 };

struct GemvParams {
  const uint16_t* W;      // [N][K] bf16 (the gate projection for kEpiGateUp)
  const uint16_t* W2;     // kEpiGateUp: the up projection [N][K]
  const float* x;         // kInNorm / kInF32: [B][K] fp32
  const uint16_t* xb;     // kInBf16: [B][K] bf16
  const float* gamma;     // kInNorm: [K]
  uint16_t* q;            // kEpiQKV: [B][Hq*128] bf16
  uint16_t* kn;           // kEpiQKV: [B][Hkv*128]
  uint16_t* vn;
  float* resid;           // kEpiResid: [B][N], += W a
  uint16_t* act;          // kEpiGateUp: [B][N] bf16
  float* logits;          // kEpiLogits: [B][N]
  int B, N, K, Hq, Hkv, n_tiles;
};

__device__ __forceinline__ uint4 ldg_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(reinterpret_cast<uint64_t>(p)));
  return v;
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Weight chunk of 32 K values for one tile: rows g and g + 8 of this lane, 8 values each.
struct WChunk {
  uint4 lo, hi;
};

// Two MMA k-steps over one 32-value chunk: physical K offsets 8c .. 8c+7 of the lane hold the
// logical k-step 0 values {2c, 2c+1 | 2c+8, 2c+9} at 8c+0..3 and k-step 1 at 8c+4..7.
__device__ __forceinline__ void chunk_mma(float (&acc)[4], const WChunk& w, const uint4& xs) {
  const uint32_t a0[4] = {w.lo.x, w.hi.x, w.lo.y, w.hi.y};
  const uint32_t a1[4] = {w.lo.z, w.hi.z, w.lo.w, w.hi.w};
  mma_bf16_16816(acc, a0, xs.x, xs.y);
  mma_bf16_16816(acc, a1, xs.z, xs.w);
}

template <int EPI, int IN>
__global__ void __launch_bounds__(kBThreads, 2) bb_gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(16) uint8_t bsm[];
  const int K = p.K, ldx = K + kPad;
  uint16_t* xs = reinterpret_cast<uint16_t*>(bsm);                        // [kMaxB][K + kPad]
  float* red = reinterpret_cast<float*>(bsm + (size_t)kMaxB * ldx * 2);  // [kBW][2][16][8]
  __shared__ float s_inv[kMaxB];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const size_t tile_bytes = (size_t)kTile * K * 2;

  // weights never depend on the previous kernel: pull this CTA's tiles toward L2 first
  // (the first two tiles only: a large projection, such as the LM head, would not fit in L2)
  if (tid == 0) {
    for (int t = blockIdx.x, i = 0; t < p.n_tiles && i < 2; t += gridDim.x, ++i) {
      prefetch_l2_bulk(p.W + (size_t)t * kTile * K, (uint32_t)tile_bytes);
      if (EPI == kEpiGateUp) prefetch_l2_bulk(p.W2 + (size_t)t * kTile * K, (uint32_t)tile_bytes);
    }
  }
  grid_dependency_wait();
  grid_dependents_launch();

  // ---- the bf16 input vectors of the batch, in shared memory (rows >= B are zero)
  if (IN == kInNorm) {
    if (warp < kMaxB) {
      float ss = 0.f;
      if (warp < p.B)
        for (int k = lane; k < K; k += 32) {
          const float v = p.x[(size_t)warp * K + k];
          ss = fmaf(v, v, ss);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_inv[warp] = rsqrtf(ss / (float)K + kEps);
    }
    __syncthreads();
  }
  for (int i = tid; i < kMaxB * (K / 2); i += kBThreads) {
    const int b = i / (K / 2), k = 2 * (i - b * (K / 2));
    uint32_t w = 0u;
    if (b < p.B) {
      if (IN == kInBf16) {
        w = *reinterpret_cast<const uint32_t*>(p.xb + (size_t)b * K + k);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(p.x + (size_t)b * K + k);
        float v0 = v.x, v1 = v.y;
        if (IN == kInNorm) {
          v0 = v0 * s_inv[b] * p.gamma[k];
          v1 = v1 * s_inv[b] * p.gamma[k + 1];
        }
        w = (uint32_t)f32_to_bf16_bits(v0) | ((uint32_t)f32_to_bf16_bits(v1) << 16);
      }
    }
    *reinterpret_cast<uint32_t*>(xs + (size_t)b * ldx + k) = w;
  }
  __syncthreads();

  const int kw = K / kBW;                  // K values per warp
  const int nch = kw / 32;                 // chunks per warp (a multiple of 2)
  const uint16_t* xrow = xs + (size_t)g * ldx + warp * kw + 8 * c;
  for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
    const int r0 = t * kTile;
    const uint16_t* wr0 = p.W + (size_t)(r0 + g) * K + warp * kw + 8 * c;
    const uint16_t* wr8 = wr0 + (size_t)8 * K;
    const uint16_t* ur0 = EPI == kEpiGateUp ? p.W2 + (size_t)(r0 + g) * K + warp * kw + 8 * c : nullptr;
    const uint16_t* ur8 = EPI == kEpiGateUp ? ur0 + (size_t)8 * K : nullptr;
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    // two chunks in registers while the next two load
    WChunk w[2], u[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      w[j].lo = ldg_stream(wr0 + 32 * j);
      w[j].hi = ldg_stream(wr8 + 32 * j);
      if (EPI == kEpiGateUp) {
        u[j].lo = ldg_stream(ur0 + 32 * j);
        u[j].hi = ldg_stream(ur8 + 32 * j);
      }
    }
    for (int ch = 0; ch < nch; ch += 2) {
      WChunk wn[2], un[2];
      const bool more = ch + 2 < nch;
      if (more) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          wn[j].lo = ldg_stream(wr0 + 32 * (ch + 2 + j));
          wn[j].hi = ldg_stream(wr8 + 32 * (ch + 2 + j));
          if (EPI == kEpiGateUp) {
            un[j].lo = ldg_stream(ur0 + 32 * (ch + 2 + j));
            un[j].hi = ldg_stream(ur8 + 32 * (ch + 2 + j));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xrow + 32 * (ch + j));
        chunk_mma(acc, w[j], xv);
        if (EPI == kEpiGateUp) chunk_mma(accu, u[j], xv);
      }
      if (more) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          w[j] = wn[j];
          if (EPI == kEpiGateUp) u[j] = un[j];
        }
      }
    }
    // ---- reduce the warps' K slices in warp order; lane (g, c) holds rows g, g + 8 and
    // sequences 2c, 2c + 1
    float* rw = red + (size_t)warp * 2 * kTile * kMaxB;
    rw[g * kMaxB + 2 * c] = acc[0];
    rw[g * kMaxB + 2 * c + 1] = acc[1];
    rw[(g + 8) * kMaxB + 2 * c] = acc[2];
    rw[(g + 8) * kMaxB + 2 * c + 1] = acc[3];
    if (EPI == kEpiGateUp) {
      rw[kTile * kMaxB + g * kMaxB + 2 * c] = accu[0];
      rw[kTile * kMaxB + g * kMaxB + 2 * c + 1] = accu[1];
      rw[kTile * kMaxB + (g + 8) * kMaxB + 2 * c] = accu[2];
      rw[kTile * kMaxB + (g + 8) * kMaxB + 2 * c + 1] = accu[3];
    }
    __syncthreads();
    if (tid < kTile * kMaxB) {
      const int row = tid / kMaxB, b = tid - row * kMaxB;
      float y = 0.f, yu = 0.f;
#pragma unroll
      for (int ww = 0; ww < kBW; ++ww) {
        y += red[(size_t)ww * 2 * kTile * kMaxB + tid];
        if (EPI == kEpiGateUp) yu += red[(size_t)ww * 2 * kTile * kMaxB + kTile * kMaxB + tid];
      }
      const int n = r0 + row;
      if (b < p.B) {
        if (EPI == kEpiQKV) {
          const int nq = p.Hq * 128, nk = p.Hkv * 128;
          const uint16_t v = f32_to_bf16_bits(y);
          if (n < nq) p.q[(size_t)b * nq + n] = v;
          else if (n < nq + nk) p.kn[(size_t)b * nk + (n - nq)] = v;
          else p.vn[(size_t)b * nk + (n - nq - nk)] = v;
        } else if (EPI == kEpiResid) {
          p.resid[(size_t)b * p.N + n] += y;
        } else if (EPI == kEpiGateUp) {
          const float sl = y / (1.0f + expf(-y));
          p.act[(size_t)b * p.N + n] = f32_to_bf16_bits(sl * yu);
        } else {
          p.logits[(size_t)b * p.N + n] = y;
        }
      }
    }
    __syncthreads();
  }
}

// x[b] <- src[b] (the residual stream of a pass starts from E(x_t)).
__global__ void bb_copy_kernel(const float4* src, float4* dst, int n4) {
  grid_dependency_wait();
  grid_dependents_launch();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x) dst[i] = src[i];
}

// h[b] = RMSNorm(x[b]) * gamma (fp32); one CTA per sequence.
__global__ void __launch_bounds__(1024) bb_norm_kernel(const float* x, const float* gamma, float* h, int D) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int b = blockIdx.x;
  __shared__ float red[32];
  float ss = 0.f;
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    const float v = x[(size_t)b * D + k];
    ss = fmaf(v, v, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) red[0] = rsqrtf(t / (float)D + kEps);
  }
  __syncthreads();
  const float inv = red[0];
  for (int k = threadIdx.x; k < D; k += blockDim.x) h[(size_t)b * D + k] = x[(size_t)b * D + k] * inv * gamma[k];
}

// token[b] = the smallest index of the largest logit; emb[b] = fp32(E[token[b]]).  One CTA per
// sequence.  If token_in is given, the argmax is skipped and its tokens are embedded.
__global__ void __launch_bounds__(1024) bb_argmax_embed_kernel(const float* logits, int V,
                                                               const int32_t* token_in,
                                                               int32_t* token, const uint16_t* E,
                                                               float* emb, int D) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int b = blockIdx.x;
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int s_tok;
  if (token_in) {
    if (threadIdx.x == 0) {
      const int t = token_in[b];
      s_tok = (t >= 0 && t < V) ? t : 0;
    }
  } else {
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
      const float v = logits[(size_t)b * V + i];
      if (v > best) {   // i increases per thread: the first maximum is kept
        best = v;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) {
        best = ov;
        bi = oi;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      sv[threadIdx.x >> 5] = best;
      si[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int nw = blockDim.x >> 5;
      best = threadIdx.x < nw ? sv[threadIdx.x] : -INFINITY;
      bi = threadIdx.x < nw ? si[threadIdx.x] : 0x7fffffff;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) {
          best = ov;
          bi = oi;
        }
      }
      if (threadIdx.x == 0) s_tok = (bi >= 0 && bi < V) ? bi : 0;
    }
  }
  __syncthreads();
  const int t = s_tok;
  if (threadIdx.x == 0) token[b] = t;
  for (int k = threadIdx.x; k < D; k += blockDim.x)
    emb[(size_t)b * D + k] = __uint_as_float((uint32_t)E[(size_t)t * D + k] << 16);
}

int g_bb_smem_optin = 0;

template <int EPI, int IN>
oda_status launch_gemv(oda_ctx* ctx, const GemvParams& p, cudaStream_t s) {
  const size_t smem = (size_t)kMaxB * (p.K + kPad) * 2 + (size_t)kBW * 2 * kTile * kMaxB * 4;
  if ((int)smem > g_bb_smem_optin)
    return set_error(ODA_ERR_UNSUPPORTED, "backbone: input width %d needs more shared memory", p.K);
  oda_status st = check_cuda(cudaFuncSetAttribute(bb_gemv_kernel<EPI, IN>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                             "cudaFuncSetAttribute(backbone)");
  if (st != ODA_OK) return st;
  int occ = 0;
  st = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, bb_gemv_kernel<EPI, IN>, kBThreads, smem),
                  "cudaOccupancyMaxActiveBlocksPerMultiprocessor(backbone)");
  if (st != ODA_OK) return st;
  const int grid = std::max(1, std::min(p.n_tiles, ctx->n_sms * std::max(1, occ)));
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(kBThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = ctx->cfg.overlap_layers ? 1 : 0;
  st = check_cuda(cudaLaunchKernelEx(&lc, bb_gemv_kernel<EPI, IN>, p), "backbone projection launch");
  ctx->prev_attention = (st == ODA_OK);
  return st;
}

template <class K, class... Args>
oda_status launch_small(oda_ctx* ctx, K kernel, dim3 grid, dim3 block, cudaStream_t s, const char* what,
                        Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = ctx->cfg.overlap_layers ? 1 : 0;
  oda_status st = check_cuda(cudaLaunchKernelEx(&lc, kernel, args...), what);
  ctx->prev_attention = (st == ODA_OK);
  return st;
}

oda_status check_shapes(oda_ctx* ctx, int K, int N, const char* who) {
  const oda_config& cf = ctx->cfg;
  if (cf.batch > kMaxB) return set_error(ODA_ERR_UNSUPPORTED, "%s: batch above %d", who, kMaxB);
  if (K < 512 || K % 512 != 0 || N < kTile || N % kTile != 0)
    return set_error(ODA_ERR_UNSUPPORTED, "%s: need K a multiple of 512 and N of 16 (K=%d N=%d)", who, K, N);
  if (g_bb_smem_optin == 0) {
    int dev = 0;
    oda_status st = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
    if (st == ODA_OK)
      st = check_cuda(cudaDeviceGetAttribute(&g_bb_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev),
                      "cudaDeviceGetAttribute");
    if (st != ODA_OK) return st;
  }
  return ODA_OK;
}

bool misaligned(const void* a) { return (reinterpret_cast<uintptr_t>(a) & 15) != 0; }

}  // namespace

oda_status launch_bb_qkv(oda_ctx* ctx, const oda_bb_layer* w, const float* x, void* q, void* k_new,
                         void* v_new, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128, N = (cf.n_q_heads + 2 * cf.n_kv_heads) * 128;
  if (!w || !w->attn_norm || !w->w_qkv || !x || !q || !k_new || !v_new)
    return set_error(ODA_ERR_INVALID_ARG, "bb_qkv: null pointer argument");
  if (misaligned(w->w_qkv) || misaligned(x))
    return set_error(ODA_ERR_INVALID_ARG, "bb_qkv: weights and x must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, N, "bb_qkv");
  if (st != ODA_OK) return st;
  GemvParams p = {};
  p.W = static_cast<const uint16_t*>(w->w_qkv);
  p.x = x;
  p.gamma = w->attn_norm;
  p.q = static_cast<uint16_t*>(q);
  p.kn = static_cast<uint16_t*>(k_new);
  p.vn = static_cast<uint16_t*>(v_new);
  p.B = cf.batch;
  p.N = N;
  p.K = D;
  p.Hq = cf.n_q_heads;
  p.Hkv = cf.n_kv_heads;
  p.n_tiles = N / kTile;
  return launch_gemv<kEpiQKV, kInNorm>(ctx, p, s);
}

oda_status launch_bb_attn_out(oda_ctx* ctx, const oda_bb_layer* w, const float* o, float* x, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128;
  if (!w || !w->w_o || !o || !x) return set_error(ODA_ERR_INVALID_ARG, "bb_attn_out: null pointer argument");
  if (misaligned(w->w_o) || misaligned(o) || misaligned(x))
    return set_error(ODA_ERR_INVALID_ARG, "bb_attn_out: weights, o and x must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, D, "bb_attn_out");
  if (st != ODA_OK) return st;
  GemvParams p = {};
  p.W = static_cast<const uint16_t*>(w->w_o);
  p.x = o;
  p.resid = x;
  p.B = cf.batch;
  p.N = D;
  p.K = D;
  p.n_tiles = D / kTile;
  return launch_gemv<kEpiResid, kInF32>(ctx, p, s);
}

oda_status launch_bb_mlp(oda_ctx* ctx, const oda_bb_layer* w, float* x, void* act, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128, F = w ? w->ffn : 0;
  if (!w || !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down || !x || !act)
    return set_error(ODA_ERR_INVALID_ARG, "bb_mlp: null pointer argument");
  if (misaligned(w->w_gate) || misaligned(w->w_up) || misaligned(w->w_down) || misaligned(x) ||
      misaligned(act))
    return set_error(ODA_ERR_INVALID_ARG, "bb_mlp: weights, x and act must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, F, "bb_mlp(gate/up)");
  if (st == ODA_OK) st = check_shapes(ctx, F, D, "bb_mlp(down)");
  if (st != ODA_OK) return st;
  GemvParams p = {};
  p.W = static_cast<const uint16_t*>(w->w_gate);
  p.W2 = static_cast<const uint16_t*>(w->w_up);
  p.x = x;
  p.gamma = w->mlp_norm;
  p.act = static_cast<uint16_t*>(act);
  p.B = cf.batch;
  p.N = F;
  p.K = D;
  p.n_tiles = F / kTile;
  st = launch_gemv<kEpiGateUp, kInNorm>(ctx, p, s);
  if (st != ODA_OK) return st;
  GemvParams d = {};
  d.W = static_cast<const uint16_t*>(w->w_down);
  d.xb = static_cast<const uint16_t*>(act);
  d.resid = x;
  d.B = cf.batch;
  d.N = D;
  d.K = F;
  d.n_tiles = D / kTile;
  return launch_gemv<kEpiResid, kInBf16>(ctx, d, s);
}

oda_status launch_bb_begin(oda_ctx* ctx, const float* emb, float* x, cudaStream_t s) {
  const int D = ctx->cfg.n_q_heads * 128;
  if (!emb || !x) return set_error(ODA_ERR_INVALID_ARG, "bb_begin: null pointer argument");
  if (misaligned(emb) || misaligned(x)) return set_error(ODA_ERR_INVALID_ARG, "bb_begin: buffers must be 16-byte aligned");
  const int n4 = ctx->cfg.batch * D / 4;
  return launch_small(ctx, bb_copy_kernel, dim3((n4 + 255) / 256), dim3(256), s, "bb_begin launch",
                      reinterpret_cast<const float4*>(emb), reinterpret_cast<float4*>(x), n4);
}

oda_status launch_bb_final_norm(oda_ctx* ctx, const float* gamma, const float* x, float* h, cudaStream_t s) {
  const int D = ctx->cfg.n_q_heads * 128;
  if (!gamma || !x || !h) return set_error(ODA_ERR_INVALID_ARG, "bb_final_norm: null pointer argument");
  return launch_small(ctx, bb_norm_kernel, dim3(ctx->cfg.batch), dim3(1024), s, "bb_final_norm launch",
                      x, gamma, h, D);
}

oda_status launch_bb_lm_head(oda_ctx* ctx, const void* embed, int32_t vocab, const float* h,
                             float* logits, int32_t* token, float* next_emb, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128;
  if (!embed || !h || !logits || !token || !next_emb)
    return set_error(ODA_ERR_INVALID_ARG, "bb_lm_head: null pointer argument");
  if (misaligned(embed) || misaligned(h)) return set_error(ODA_ERR_INVALID_ARG, "bb_lm_head: embed and h must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, vocab, "bb_lm_head");
  if (st != ODA_OK) return st;
  GemvParams p = {};
  p.W = static_cast<const uint16_t*>(embed);
  p.x = h;
  p.logits = logits;
  p.B = cf.batch;
  p.N = vocab;
  p.K = D;
  p.n_tiles = vocab / kTile;
  st = launch_gemv<kEpiLogits, kInF32>(ctx, p, s);
  if (st != ODA_OK) return st;
  return launch_small(ctx, bb_argmax_embed_kernel, dim3(cf.batch), dim3(1024), s, "bb_argmax launch",
                      (const float*)logits, (int)vocab, (const int32_t*)nullptr, token,
                      static_cast<const uint16_t*>(embed), next_emb, D);
}

oda_status launch_bb_embed(oda_ctx* ctx, const void* embed, int32_t vocab, const int32_t* token,
                           float* emb, cudaStream_t s) {
  const int D = ctx->cfg.n_q_heads * 128;
  if (!embed || !token || !emb || vocab < 1) return set_error(ODA_ERR_INVALID_ARG, "bb_embed: bad argument");
  // the token buffer is read, and rewritten with the (range-checked) token it used
  return launch_small(ctx, bb_argmax_embed_kernel, dim3(ctx->cfg.batch), dim3(1024), s, "bb_embed launch",
                      (const float*)nullptr, (int)vocab, token, const_cast<int32_t*>(token),
                      static_cast<const uint16_t*>(embed), emb, D);
}

}  // namespace oda
