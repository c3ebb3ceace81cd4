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
constexpr int kTile = 16;              // output rows per tile
constexpr int kMaxB = 8;               // sequences: the MMA's N
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
  int32_t* err;
  int B, N, K, Hq, Hkv, n_tiles;
  int kst;                // K values per stage (a K chunk of one tile)
  int ring;               // stages in the ring
};

constexpr int kXPad = 8;            // bf16 padding of an input row (rows 4 banks apart)
constexpr int kRowPad = 8;          // bf16 padding of a staged weight row
constexpr int kGThreads = (kBW + 1) * 32;   // 8 consumer warps + 1 producer warp
constexpr int kMaxRing = 6;
constexpr uint64_t kGWaitNs = 2000000000ull;

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kBW * 32) : "memory");
}

// Persistent projection: one CTA per SM takes tiles t = blockIdx.x, + gridDim.x, ...  A producer
// warp streams each tile's rows, K chunk by K chunk, through a ring of shared-memory stages with
// one bulk copy per row segment (completion counted on the stage's mbarrier); it only reads
// weights, so it fills the ring before the previous kernel has finished.  The 8 consumer warps
// each take 1/8 of every chunk's columns: A fragments of the 16 rows by ldmatrix, B fragments of
// the bf16 inputs (in shared memory) by ldmatrix, mma.sync bf16 -> fp32.  At the end of a tile
// the warps' partial sums are added in warp order and the epilogue writes the outputs.
template <int EPI, int IN>
__global__ void __launch_bounds__(kGThreads, 1) bb_gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(128) uint8_t bsm[];
  constexpr int kRows = EPI == kEpiGateUp ? 2 * kTile : kTile;
  const int K = p.K, kst = p.kst, R = p.ring, nck = K / kst;
  const int ldx = K + kXPad, ldw = kst + kRowPad;
  const size_t stage_bytes = (size_t)kRows * ldw * 2;
  uint8_t* stages = bsm;
  uint16_t* xs = reinterpret_cast<uint16_t*>(bsm + R * stage_bytes);              // [8][K + pad]
  float* red = reinterpret_cast<float*>(bsm + R * stage_bytes + (size_t)kMaxB * ldx * 2);
  __shared__ __align__(8) uint64_t full[kMaxRing];
  __shared__ __align__(8) uint64_t empty[kMaxRing];
  __shared__ float s_inv[kMaxB];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kBW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kBW) {
    // ---- producer: every (tile, chunk) of this CTA in order
    int k = 0;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
      for (int ch = 0; ch < nck; ++ch, ++k) {
        const int s = k % R;
        if (k >= R && !mbar_wait_bounded(&empty[s], (uint32_t)(k / R - 1) & 1u, kGWaitNs)) {
          if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
          return;
        }
        if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(kRows * kst * 2));
        __syncwarp();
        if (lane < kRows) {
          const uint16_t* src = (EPI == kEpiGateUp && lane >= kTile)
                                    ? p.W2 + (size_t)(t * kTile + lane - kTile) * K + ch * kst
                                    : p.W + (size_t)(t * kTile + lane) * K + ch * kst;
          fence_proxy_async_smem();
          bulk_load(stages + s * stage_bytes + (size_t)lane * ldw * 2, src, (uint32_t)(kst * 2), &full[s]);
        }
      }
    }
    return;
  }

  // ---- consumers
  grid_dependency_wait();
  grid_dependents_launch();
  if (IN == kInNorm) {
    if (warp < kMaxB) {
      float ss = 0.f;
      if (warp < p.B)
        for (int kk = 4 * lane; kk < K; kk += 128) {
          const float4 v = *reinterpret_cast<const float4*>(p.x + (size_t)warp * K + kk);
          ss = fmaf(v.x, v.x, ss);
          ss = fmaf(v.y, v.y, ss);
          ss = fmaf(v.z, v.z, ss);
          ss = fmaf(v.w, v.w, ss);
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_inv[warp] = rsqrtf(ss / (float)K + kEps);
    }
    consumers_sync();
  }
  for (int i = tid; i < kMaxB * (K / 2); i += kBW * 32) {
    const int b = i / (K / 2), kk = 2 * (i - b * (K / 2));
    uint32_t w = 0u;
    if (b < p.B) {
      if (IN == kInBf16) {
        w = *reinterpret_cast<const uint32_t*>(p.xb + (size_t)b * K + kk);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(p.x + (size_t)b * K + kk);
        float v0 = v.x, v1 = v.y;
        if (IN == kInNorm) {
          v0 = v0 * s_inv[b] * p.gamma[kk];
          v1 = v1 * s_inv[b] * p.gamma[kk + 1];
        }
        w = (uint32_t)f32_to_bf16_bits(v0) | ((uint32_t)f32_to_bf16_bits(v1) << 16);
      }
    }
    *reinterpret_cast<uint32_t*>(xs + (size_t)b * ldx + kk) = w;
  }
  consumers_sync();

  const int g = lane >> 2, c = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int kw = kst / kBW;                      // columns of a chunk per warp (multiple of 16)
  const uint32_t xs_base = smem_u32(xs);
  // ldmatrix rows: A from the staged weight rows, B from the input rows (batch g)
  const int arow = ((mi & 1) << 3) + rr, acol = (mi >> 1) << 3;
  const int brow = rr, bcol = mi << 3;
  int k = 0;
  for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ch = 0; ch < nck; ++ch, ++k) {
      const int s = k % R;
      if (!mbar_wait_bounded(&full[s], (uint32_t)(k / R) & 1u, kGWaitNs)) {
        if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
      }
      const uint32_t sb = smem_u32(stages + s * stage_bytes);
      const int c0 = warp * kw;                  // first column of this warp in the chunk
#pragma unroll 4
      for (int kk = 0; kk < kw; kk += 32) {
        uint32_t xb4[4];
        ldsm_x4(xb4, xs_base + ((brow * ldx) + ch * kst + c0 + kk + bcol) * 2);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t a[4];
          ldsm_x4(a, sb + ((arow * ldw) + c0 + kk + 16 * h + acol) * 2);
          mma_bf16_16816(acc, a, xb4[2 * h], xb4[2 * h + 1]);
          if (EPI == kEpiGateUp) {
            uint32_t au[4];
            ldsm_x4(au, sb + (((arow + kTile) * ldw) + c0 + kk + 16 * h + acol) * 2);
            mma_bf16_16816(accu, au, xb4[2 * h], xb4[2 * h + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // ---- the warps' column shares, added in warp order; lane (g, c) holds rows g, g + 8 and
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
    consumers_sync();
    if (tid < kTile * kMaxB) {
      const int row = tid / kMaxB, b = tid - row * kMaxB;
      float y = 0.f, yu = 0.f;
#pragma unroll
      for (int ww = 0; ww < kBW; ++ww) {
        y += red[(size_t)ww * 2 * kTile * kMaxB + tid];
        if (EPI == kEpiGateUp) yu += red[(size_t)ww * 2 * kTile * kMaxB + kTile * kMaxB + tid];
      }
      const int n = t * kTile + row;
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
    consumers_sync();
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

// token[b] = the smallest index of the largest logit; emb[b] = fp32(E[token[b]]).  Grid (slices,
// B): each CTA finds the first maximum of its slice of the logits; the CTA completing sequence b
// (a completion counter, no waiting) takes the first maximum over the slices in slice order and
// writes the token and its embedding row.  With token_in (one slice), the given tokens are
// embedded instead (a token outside [0, V) is taken as 0).
__global__ void __launch_bounds__(256) bb_argmax_embed_kernel(const float* logits, int V,
                                                              const int32_t* token_in,
                                                              int32_t* token, const uint16_t* E,
                                                              float* emb, int D, float* part_v,
                                                              int32_t* part_i, int32_t* cnt) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int sl = blockIdx.x, nsl = gridDim.x, b = blockIdx.y;
  __shared__ float sv[8];
  __shared__ int si[8];
  __shared__ int s_tok, s_last;
  auto better = [](float v, int i, float bv, int bi) { return v > bv || (v == bv && i < bi); };
  if (token_in) {
    if (threadIdx.x == 0) {
      const int t = token_in[b];
      s_tok = (t >= 0 && t < V) ? t : 0;
    }
  } else {
    const int lo = (int)((long long)sl * V / nsl), hi = (int)((long long)(sl + 1) * V / nsl);
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
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
      if (better(ov, oi, best, bi)) {
        best = ov;
        bi = oi;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      sv[threadIdx.x >> 5] = best;
      si[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
        if (better(sv[w], si[w], best, bi)) {
          best = sv[w];
          bi = si[w];
        }
      if (nsl > 1) {
        part_v[(size_t)b * nsl + sl] = best;
        part_i[(size_t)b * nsl + sl] = bi;
        __threadfence();
        s_last = atomicAdd(&cnt[b], 1) == nsl - 1;
        if (s_last) {
          __threadfence();
          best = -INFINITY;
          bi = 0x7fffffff;
          for (int j = 0; j < nsl; ++j) {
            const float v = __ldcg(part_v + (size_t)b * nsl + j);
            const int i = __ldcg(part_i + (size_t)b * nsl + j);
            if (better(v, i, best, bi)) {
              best = v;
              bi = i;
            }
          }
          cnt[b] = 0;
        }
      } else {
        s_last = 1;
      }
      s_tok = (bi >= 0 && bi < V) ? bi : 0;
    }
    __syncthreads();
    if (!s_last) return;
  }
  __syncthreads();
  const int t = s_tok;
  if (threadIdx.x == 0) token[b] = t;
  for (int kk = threadIdx.x; kk < D; kk += blockDim.x)
    emb[(size_t)b * D + kk] = __uint_as_float((uint32_t)E[(size_t)t * D + kk] << 16);
}

int g_bb_smem_optin = 0;

template <int EPI, int IN>
oda_status launch_gemv(oda_ctx* ctx, GemvParams p, cudaStream_t s) {
  constexpr int rows = EPI == kEpiGateUp ? 2 * kTile : kTile;
  p.err = ctx->err;
  // a stage of about 32 KiB: 1024 columns of 16 rows, or 512 of the gate and up rows together
  p.kst = (EPI != kEpiGateUp && p.K % 1024 == 0) ? 1024 : 512;
  const size_t stage = (size_t)rows * (p.kst + kRowPad) * 2;
  const size_t fixed = (size_t)kMaxB * (p.K + kXPad) * 2 + (size_t)kBW * 2 * kTile * kMaxB * 4;
  const long long room = (long long)g_bb_smem_optin - 1024 - (long long)fixed;
  p.ring = (int)std::min<long long>(kMaxRing, room / (long long)stage);
  if (p.ring < 2)
    return set_error(ODA_ERR_UNSUPPORTED, "backbone: input width %d needs more shared memory", p.K);
  const size_t smem = p.ring * stage + fixed;
  oda_status st = check_cuda(cudaFuncSetAttribute(bb_gemv_kernel<EPI, IN>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                             "cudaFuncSetAttribute(backbone)");
  if (st != ODA_OK) return st;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(std::min(p.n_tiles, ctx->n_sms));
  lc.blockDim = dim3(kGThreads);
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
  const int nsl = std::max(1, std::min(64, vocab / 2048));
  float* part_v = ctx->bb_part;
  int32_t* part_i = reinterpret_cast<int32_t*>(ctx->bb_part + (size_t)cf.batch * nsl);
  return launch_small(ctx, bb_argmax_embed_kernel, dim3(nsl, cf.batch), dim3(256), s, "bb_argmax launch",
                      (const float*)logits, (int)vocab, (const int32_t*)nullptr, token,
                      static_cast<const uint16_t*>(embed), next_emb, D, part_v, part_i, ctx->bb_cnt);
}

oda_status launch_bb_embed(oda_ctx* ctx, const void* embed, int32_t vocab, const int32_t* token,
                           float* emb, cudaStream_t s) {
  const int D = ctx->cfg.n_q_heads * 128;
  if (!embed || !token || !emb || vocab < 1) return set_error(ODA_ERR_INVALID_ARG, "bb_embed: bad argument");
  // the token buffer is read, and rewritten with the (range-checked) token it used
  return launch_small(ctx, bb_argmax_embed_kernel, dim3(1, ctx->cfg.batch), dim3(256), s, "bb_embed launch",
                      (const float*)nullptr, (int)vocab, token, const_cast<int32_t*>(token),
                      static_cast<const uint16_t*>(embed), emb, D, ctx->bb_part,
                      reinterpret_cast<int32_t*>(ctx->bb_part), ctx->bb_cnt);
}

}  // namespace oda
