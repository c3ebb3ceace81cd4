// Training-side arithmetic of the recall head: labels, Huber loss and the gradient of the loss
// with respect to every head parameter, fp32.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.1 eq. g_t (gain), §2.2
// eqs. d_t and y_t (penalised gain, label) and eq. L(psi) (mean Huber-1 error over the valid
// positions E; only the recall head receives gradients).  The head is the reading documented in
// head.cu: towers u_i = SiLU(W_i (RMSNorm(x_i) gamma_i) + b_i), interaction z, fusion
// f0 = W_f z + b_f + mean(u), two residual gated FFN blocks, q = w_o . (RMSNorm(f2) gamma_o) + b_o.
//
// Design: a training step is a handful of weight-streaming passes at batch sizes of a few
// sequences, so every matrix is touched by plain CUDA-core kernels that stream it once per pass:
//   * forward recompute (activations kept in the caller's workspace): row GEMVs split into
//     1024-column chunks, partial sums reduced in chunk order with the phase's epilogue;
//   * backward: one pass per matrix reads each weight row once, writes its gradient row
//     dW[n] = sum_b dY[b][n] X[b] and accumulates W^T dY into per-row-block partials, which a
//     second kernel sums in row-block order (with the next elementwise step fused in);
//   * small per-sequence kernels for the RMSNorm scales and backward, the labels and the loss.
// Every reduction has a fixed order, so results are deterministic.  Batch at most 16.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "internal.h"

namespace oda {
namespace {

constexpr int kGT = 1024;         // tower width
constexpr int kGF = 2048;         // FFN width
constexpr int kGZ = 9 * kGT;      // interaction width
constexpr int kCol = 1024;        // columns per chunk
constexpr int kRowsFwd = 16;      // rows per CTA in the forward GEMV (8 warps x 2)
constexpr int kRowsBwd = 16;      // rows per CTA in the backward pass
constexpr int kGB = 16;           // largest batch
constexpr float kGEps = 1e-6f;

__device__ __forceinline__ float sigm(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float silu_f(float x) { return x * sigm(x); }
__device__ __forceinline__ float silu_d(float x) {
  const float s = sigm(x);
  return s * (1.0f + x * (1.0f - s));
}
__device__ __forceinline__ float sgn(float a, float b) { return (float)((a > b) - (a < b)); }

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide sum (up to 1024 threads) in a fixed order; every thread receives the total.
__device__ float block_sum_f(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_f(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  __syncthreads();
  return t;
}

// ------------------------------------------------------------------ forward GEMV
// part[c][b][n] = sum_{k in chunk c} W[n][k] X[b][k]  for rows n of the CTA's block; X rows
// are ldx floats apart.  Grid (N / 16, K / 1024), 256 threads: warp w takes rows 2w, 2w+1, whose
// loads are all issued before the first product.
__global__ void __launch_bounds__(256) gemv_rows_kernel(const float* W, int N, int K, const float* X,
                                                        int ldx, int B, float* part) {
  extern __shared__ float xs[];   // [B][1024]
  const int rb = blockIdx.x, c = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = c * kCol;
  for (int i = threadIdx.x; i < B * kCol; i += 256) {
    const int b = i / kCol, k = i - b * kCol;
    xs[i] = X[(size_t)b * ldx + k0 + k];
  }
  __syncthreads();
  const float4* x4 = reinterpret_cast<const float4*>(xs);
  const int n0 = rb * kRowsFwd + warp * 2;
  float4 wv[2][kCol / 128];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float4* w4 = reinterpret_cast<const float4*>(W + (size_t)(n0 + r) * K + k0);
#pragma unroll
    for (int j = 0; j < kCol / 128; ++j) wv[r][j] = __ldcs(w4 + lane + 32 * j);
  }
  for (int b = 0; b < B; ++b) {
    float acc[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kCol / 128; ++j) {
      const float4 xv = x4[b * (kCol / 4) + lane + 32 * j];
#pragma unroll
      for (int r = 0; r < 2; ++r)
        acc[r] += wv[r][j].x * xv.x + wv[r][j].y * xv.y + wv[r][j].z * xv.z + wv[r][j].w * xv.w;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float t = warp_sum_f(acc[r]);
      if (lane == 0) part[((size_t)c * B + b) * N + n0 + r] = t;
    }
  }
}

// Epilogues of the forward reductions.
enum FwdEpi { kEpiTower = 0, kEpiFuse = 1, kEpiStore = 2, kEpiUp = 3, kEpiDown = 4 };

struct FwdArgs {
  const float* part;
  int nchunk, B, N;
  int epi;
  const float* bias;     // tower: b_i; fuse: b_f
  const float* u;        // fuse: [3][B][T] tower outputs
  const float* g;        // up: the gate pre-activations g [B][F] (an earlier launch)
  const float* f_in;     // down: f_j [B][T]
  float* out;            // tower: u_i; fuse: f0; store: g; up: v; down: f_{j+1}
  float* out2;           // tower: p_i (pre-activation); up: a = SiLU(g) v
};

// Sums the chunks in order and applies the epilogue; one thread per (b, n).
__global__ void fwd_reduce_kernel(const FwdArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.B * a.N) return;
  const int b = i / a.N, n = i - b * a.N;
  float acc = 0.f;
  for (int c = 0; c < a.nchunk; ++c) acc += a.part[((size_t)c * a.B + b) * a.N + n];
  switch (a.epi) {
    case kEpiTower: {
      const float p = acc + a.bias[n];
      a.out2[i] = p;
      a.out[i] = silu_f(p);
      break;
    }
    case kEpiFuse: {
      const float mean = (a.u[((size_t)0 * a.B + b) * kGT + n] + a.u[((size_t)1 * a.B + b) * kGT + n] +
                          a.u[((size_t)2 * a.B + b) * kGT + n]) / 3.0f;
      a.out[i] = acc + a.bias[n] + mean;
      break;
    }
    case kEpiStore:
      a.out[i] = acc;
      break;
    case kEpiUp:
      a.out[i] = acc;
      a.out2[i] = silu_f(a.g[i]) * acc;
      break;
    default:
      a.out[i] = a.f_in[i] + acc;
      break;
  }
}

// ------------------------------------------------------------------ backward pass
// For rows [16 rb, 16 rb + 16) of W [N][K] and columns [1024 c, 1024 c + 1024):
//   dW[n][k]        = sum_b dY[b][n] X[b][k]          (each (n, k) written by one thread)
//   part[rb][b][k]  = sum_{n in the block} W[n][k] dY[b][n]
// 256 threads; thread t owns the four columns 1024 c + 4t .. +3.  Grid (N / 16, K / 1024).  The
// weight loads of 8 rows are issued before their products; with batches up to 8 two CTAs share
// an SM, so one CTA's loads overlap the other's products and stores.
template <int BM>
__global__ void __launch_bounds__(256, BM <= 8 ? 2 : 1) bwd_rows_kernel(const float* W, int N, int K, const float* dY,
                                                       int ldy, const float* X, int ldx, int B,
                                                       float* dW, float* part) {
  __shared__ float dys[kRowsBwd * BM];   // [row][b]
  const int rb = blockIdx.x, t = threadIdx.x;
  const int n0 = rb * kRowsBwd, col = blockIdx.y * kCol + 4 * t;
  for (int i = t; i < kRowsBwd * B; i += 256) {
    const int r = i / B, b = i - r * B;
    dys[r * BM + b] = dY[(size_t)b * ldy + n0 + r];
  }
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 x[BM], acc[BM];
#pragma unroll
  for (int b = 0; b < BM; ++b) {
    x[b] = b < B ? *reinterpret_cast<const float4*>(X + (size_t)b * ldx + col) : zero;
    acc[b] = zero;
  }
  __syncthreads();
  constexpr int RB = 8;
#pragma unroll 1
  for (int r0 = 0; r0 < kRowsBwd; r0 += RB) {
    float4 wv[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r)
      wv[r] = __ldcs(reinterpret_cast<const float4*>(W + (size_t)(n0 + r0 + r) * K + col));
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const float4 w = wv[r];
      float4 g = zero;
#pragma unroll
      for (int b = 0; b < BM; ++b) {
        if (b < B) {
          const float d = dys[(r0 + r) * BM + b];
          g.x += d * x[b].x;
          g.y += d * x[b].y;
          g.z += d * x[b].z;
          g.w += d * x[b].w;
          acc[b].x += d * w.x;
          acc[b].y += d * w.y;
          acc[b].z += d * w.z;
          acc[b].w += d * w.w;
        }
      }
      __stcs(reinterpret_cast<float4*>(dW + (size_t)(n0 + r0 + r) * K + col), g);
    }
  }
#pragma unroll
  for (int b = 0; b < BM; ++b)
    if (b < B) *reinterpret_cast<float4*>(part + ((size_t)rb * B + b) * K + col) = acc[b];
}

enum BwdEpi { kBwdStore = 0, kBwdGate = 1 };

struct BwdArgs {
  const float* part;     // [nrb][B][K]
  const float* part2;    // optional second set [nrb2][B][K], added after the first
  int nrb, nrb2, B, K;
  int epi;
  const float* g;        // gate: g [B][F]
  const float* v;        // gate: v [B][F]
  float* out;            // store: the sum; gate: dg
  float* out2;           // gate: dv
};

// Sums the partials and applies the epilogue (gate: da -> dg = da v SiLU'(g), dv = da
// SiLU(g)).  A CTA of 256 takes 32 consecutive outputs (b, k); its eight warps each sum every
// eighth row block (the second set continues the numbering), and warp 0 adds the eight slices
// in order: a fixed order, with eight times the loads in flight of one thread per output.
__global__ void __launch_bounds__(256) bwd_reduce_kernel(const BwdArgs a) {
  __shared__ float sl[8][33];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = blockIdx.x * 32 + lane;   // B * K is a multiple of 32
  const int b = i / a.K, k = i - b * a.K;
  float acc = 0.f;
  for (int r = w; r < a.nrb + a.nrb2; r += 8)
    acc += r < a.nrb ? a.part[((size_t)r * a.B + b) * a.K + k]
                     : a.part2[((size_t)(r - a.nrb) * a.B + b) * a.K + k];
  sl[w][lane] = acc;
  __syncthreads();
  if (w != 0) return;
  acc = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) acc += sl[j][lane];
  if (a.epi == kBwdStore) {
    a.out[i] = acc;
  } else {
    const float g = a.g[i];
    a.out[i] = acc * a.v[i] * silu_d(g);
    a.out2[i] = acc * silu_f(g);
  }
}

// ------------------------------------------------------------------ small kernels
// Per sequence (one CTA of 1024 per b): s[b] = 1 / rms(x_b), y_b = x_b s gamma.
__global__ void rms_kernel(const float* x, int K, const float* gamma, float* s, float* y) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float* xb = x + (size_t)b * K;
  float ss = 0.f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) ss += xb[k] * xb[k];
  const float sc = rsqrtf(block_sum_f(ss, red) / K + kGEps);
  if (threadIdx.x == 0) s[b] = sc;
  for (int k = threadIdx.x; k < K; k += blockDim.x) y[(size_t)b * K + k] = xb[k] * sc * gamma[k];
}

// z = [u0, u1, u2, u0 u1, u0 u2, u1 u2, |u0 - u1|, |u0 - u2|, |u1 - u2|]; one thread per (b, n).
__global__ void interaction_kernel(const float* u, int B, float* z) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * kGT) return;
  const int b = i / kGT, n = i - b * kGT;
  const float u0 = u[((size_t)0 * B + b) * kGT + n], u1 = u[((size_t)1 * B + b) * kGT + n],
              u2 = u[((size_t)2 * B + b) * kGT + n];
  float* zb = z + (size_t)b * kGZ + n;
  zb[0 * kGT] = u0;
  zb[1 * kGT] = u1;
  zb[2 * kGT] = u2;
  zb[3 * kGT] = u0 * u1;
  zb[4 * kGT] = u0 * u2;
  zb[5 * kGT] = u1 * u2;
  zb[6 * kGT] = fabsf(u0 - u1);
  zb[7 * kGT] = fabsf(u0 - u2);
  zb[8 * kGT] = fabsf(u1 - u2);
}

// Per sequence b (one CTA of 1024): the score q = w_o . (f2 s gamma_o) + b_o; keeps s_o and n_o.
__global__ void score_kernel(const float* f2, const float* gamma, const float* w_o, const float* b_o,
                             float* s_o, float* n_o, float* q) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float* fb = f2 + (size_t)b * kGT;
  float ss = 0.f;
  for (int k = threadIdx.x; k < kGT; k += blockDim.x) ss += fb[k] * fb[k];
  const float sc = rsqrtf(block_sum_f(ss, red) / kGT + kGEps);
  float dot = 0.f;
  for (int k = threadIdx.x; k < kGT; k += blockDim.x) {
    const float nv = fb[k] * sc * gamma[k];
    n_o[(size_t)b * kGT + k] = nv;
    dot += w_o[k] * nv;
  }
  dot = block_sum_f(dot, red);
  if (threadIdx.x == 0) {
    s_o[b] = sc;
    q[b] = dot + b_o[0];
  }
}

// Labels, loss and dL/dq (one thread per sequence, then thread 0 sums in order):
// g = ln p^F - ln p^L, d = g - lambda, y = sign(d) log(1 + |d|), r = q - y,
// loss = mean over valid of Huber_1(r), dq = clamp(r, -1, 1) / |E| (0 where not valid).
__global__ void labels_kernel(const float* q, const float* p_full, const float* p_local,
                              const int32_t* valid, int B, float lam, float* y, float* dq,
                              float* loss) {
  __shared__ float hub[kGB];
  __shared__ int nvalid;
  const int b = threadIdx.x;
  if (b == 0) {
    int nv = 0;
    for (int i = 0; i < B; ++i) nv += valid[i] != 0;
    nvalid = nv;
  }
  __syncthreads();
  if (b < B) {
    float yb = 0.f, d = 0.f, h = 0.f;
    if (valid[b]) {
      const float dd = (logf(p_full[b]) - logf(p_local[b])) - lam;
      yb = (dd > 0.f ? 1.f : (dd < 0.f ? -1.f : 0.f)) * log1pf(fabsf(dd));
      const float r = q[b] - yb;
      const float ar = fabsf(r);
      h = ar <= 1.f ? 0.5f * r * r : ar - 0.5f;
      d = fminf(fmaxf(r, -1.f), 1.f) / (float)nvalid;
    }
    y[b] = yb;
    dq[b] = d;
    hub[b] = h;
  }
  __syncthreads();
  if (b == 0) {
    float t = 0.f;
    for (int i = 0; i < B; ++i) t += hub[i];
    *loss = nvalid > 0 ? t / (float)nvalid : 0.f;
  }
}

// RMSNorm backward for one sequence per CTA: y = x s gamma, given dy (or, for the output
// norm, dy = dq[b] w_o): dx = s h - s^3 x (h . x) / K with h = dy gamma; dx is added to dx_out
// when `accumulate`, else stored.
__global__ void rms_backward_kernel(const float* dy, const float* dq, const float* w_o,
                                    const float* x, const float* s, const float* gamma, int K,
                                    bool accumulate, float* dx_out) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float sc = s[b];
  const float* xb = x + (size_t)b * K;
  float hx = 0.f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const float d = dy ? dy[(size_t)b * K + k] : dq[b] * w_o[k];
    hx += d * gamma[k] * xb[k];
  }
  hx = block_sum_f(hx, red);
  const float c3 = sc * sc * sc * hx / K;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const float d = dy ? dy[(size_t)b * K + k] : dq[b] * w_o[k];
    const float dx = sc * d * gamma[k] - c3 * xb[k];
    float* o = dx_out + (size_t)b * K + k;
    *o = accumulate ? *o + dx : dx;
  }
}

// Gradient of a norm weight: dgamma[k] = sum_b dy[b][k] x[b][k] s[b] (dy = dq[b] w_o for the
// output norm), sequences in order; one thread per k.
__global__ void norm_weight_grad_kernel(const float* dy, const float* dq, const float* w_o,
                                        const float* x, const float* s, int B, int K, float* dgamma) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float t = 0.f;
  for (int b = 0; b < B; ++b) {
    const float d = dy ? dy[(size_t)b * K + k] : dq[b] * w_o[k];
    t += d * x[(size_t)b * K + k] * s[b];
  }
  dgamma[k] = t;
}

// Output layer: dw_o[k] = sum_b dq[b] n_o[b][k]; db_o = sum_b dq[b].  One thread per k.
__global__ void out_grad_kernel(const float* dq, const float* n_o, int B, float* dw_o, float* db_o) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= kGT) return;
  float t = 0.f;
  for (int b = 0; b < B; ++b) t += dq[b] * n_o[(size_t)b * kGT + k];
  dw_o[k] = t;
  if (k == 0) {
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += dq[b];
    db_o[0] = s;
  }
}

// Fusion and interaction backward, one thread per (b, n): du_i = df0 / 3 + the z terms, then
// dp_i = du_i SiLU'(p_i).  sign(0) = 0 for the absolute differences.
__global__ void fuse_backward_kernel(const float* df0, const float* dz, const float* u,
                                     const float* p, int B, float* dp) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * kGT) return;
  const int b = i / kGT, n = i - b * kGT;
  const float u0 = u[((size_t)0 * B + b) * kGT + n], u1 = u[((size_t)1 * B + b) * kGT + n],
              u2 = u[((size_t)2 * B + b) * kGT + n];
  const float* d = dz + (size_t)b * kGZ + n;
  const float s01 = sgn(u0, u1), s02 = sgn(u0, u2), s12 = sgn(u1, u2);
  const float f3 = df0[i] / 3.0f;
  const float du0 = f3 + d[0] + d[3 * kGT] * u1 + d[4 * kGT] * u2 + d[6 * kGT] * s01 + d[7 * kGT] * s02;
  const float du1 = f3 + d[kGT] + d[3 * kGT] * u0 + d[5 * kGT] * u2 - d[6 * kGT] * s01 + d[8 * kGT] * s12;
  const float du2 = f3 + d[2 * kGT] + d[4 * kGT] * u0 + d[5 * kGT] * u1 - d[7 * kGT] * s02 - d[8 * kGT] * s12;
  dp[((size_t)0 * B + b) * kGT + n] = du0 * silu_d(p[((size_t)0 * B + b) * kGT + n]);
  dp[((size_t)1 * B + b) * kGT + n] = du1 * silu_d(p[((size_t)1 * B + b) * kGT + n]);
  dp[((size_t)2 * B + b) * kGT + n] = du2 * silu_d(p[((size_t)2 * B + b) * kGT + n]);
}

// Sum over sequences in order: out[k] = sum_b v[b][k] (bias gradients).  One thread per k.
__global__ void batch_sum_kernel(const float* v, int B, int K, float* out) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float t = 0.f;
  for (int b = 0; b < B; ++b) t += v[(size_t)b * K + k];
  out[k] = t;
}

// Pieces of the caller's workspace (fp32, each piece 256-byte aligned).
struct GradWs {
  float *sx, *nx, *p, *u, *z, *f, *sf, *m, *g, *v, *a, *so, *no, *dq, *dF, *dG, *dV, *dM, *dZ, *dP,
      *dN, *partA, *partB;
  size_t floats;
};

GradWs carve(float* base, int B, int D) {
  GradWs w;
  size_t o = 0;
  auto take = [&](size_t n) {
    float* q = base ? base + o : nullptr;
    o += (n + 63) & ~size_t(63);
    return q;
  };
  const size_t Bs = (size_t)B;
  w.sx = take(3 * Bs);
  w.nx = take(3 * Bs * D);
  w.p = take(3 * Bs * kGT);
  w.u = take(3 * Bs * kGT);
  w.z = take(Bs * kGZ);
  w.f = take(3 * Bs * kGT);
  w.sf = take(2 * Bs);
  w.m = take(2 * Bs * kGT);
  w.g = take(2 * Bs * kGF);
  w.v = take(2 * Bs * kGF);
  w.a = take(2 * Bs * kGF);
  w.so = take(Bs);
  w.no = take(Bs * kGT);
  w.dq = take(Bs);
  w.dF = take(Bs * kGT);
  w.dG = take(Bs * kGF);
  w.dV = take(Bs * kGF);
  w.dM = take(Bs * kGT);
  w.dZ = take(Bs * kGZ);
  w.dP = take(3 * Bs * kGT);
  w.dN = take(Bs * D);
  // backward partials: 64 row blocks of the T-row matrices over up to max(9T, D) columns, or 128
  // row blocks of the F-row matrices over T columns; forward partials are smaller
  w.partA = take((size_t)(kGT / kRowsBwd) * Bs * std::max(kGZ, D));
  w.partB = take((size_t)(kGF / kRowsBwd) * Bs * kGT);
  w.floats = o;
  return w;
}

}  // namespace

size_t recall_grad_workspace_bytes(int B, int D) {
  return carve(nullptr, B, D).floats * sizeof(float);
}

oda_status launch_recall_grad(const oda_head_weights* w, const oda_head_grads* gr, int B, int D,
                              const float* h_prev, const float* emb, const float* h_loc,
                              const float* p_full, const float* p_local, const int32_t* valid,
                              float lam, float* loss, float* q, float* y, void* workspace,
                              size_t workspace_bytes, cudaStream_t s) {
  if (!w || !gr || !h_prev || !emb || !h_loc || !p_full || !p_local || !valid || !loss || !q ||
      !y || !workspace)
    return set_error(ODA_ERR_INVALID_ARG, "recall_grad: null pointer argument");
  if (B < 1 || B > kGB)
    return set_error(ODA_ERR_UNSUPPORTED, "recall_grad: batch must be 1..%d (got %d)", kGB, B);
  if (D < kCol || D > 8192 || D % kCol != 0)
    return set_error(ODA_ERR_UNSUPPORTED, "recall_grad: head_in_dim must be a multiple of 1024 in 1024..8192");
  if (workspace_bytes < recall_grad_workspace_bytes(B, D))
    return set_error(ODA_ERR_INVALID_ARG, "recall_grad: workspace of %zu bytes, %zu needed", workspace_bytes,
                     recall_grad_workspace_bytes(B, D));
  const void* aligned[] = {workspace, h_prev, emb, h_loc, w->fuse_w, gr->fuse_w, w->tower_w[0],
                           w->tower_w[1], w->tower_w[2], gr->tower_w[0], gr->tower_w[1], gr->tower_w[2],
                           w->ffn_gate[0], w->ffn_gate[1], w->ffn_up[0], w->ffn_up[1], w->ffn_down[0],
                           w->ffn_down[1], gr->ffn_gate[0], gr->ffn_gate[1], gr->ffn_up[0], gr->ffn_up[1],
                           gr->ffn_down[0], gr->ffn_down[1]};
  for (const void* q2 : aligned)
    if (!q2 || (reinterpret_cast<uintptr_t>(q2) & 15))
      return set_error(ODA_ERR_INVALID_ARG, "recall_grad: matrices, gradients, inputs and workspace must be 16-byte aligned");
  const void* vecs[] = {w->fuse_b, w->out_norm, w->out_w, w->out_b, gr->fuse_b, gr->out_norm, gr->out_w,
                        gr->out_b, w->tower_norm[0], w->tower_norm[1], w->tower_norm[2], w->tower_b[0],
                        w->tower_b[1], w->tower_b[2], w->ffn_norm[0], w->ffn_norm[1], gr->tower_norm[0],
                        gr->tower_norm[1], gr->tower_norm[2], gr->tower_b[0], gr->tower_b[1],
                        gr->tower_b[2], gr->ffn_norm[0], gr->ffn_norm[1]};
  for (const void* q2 : vecs)
    if (!q2) return set_error(ODA_ERR_INVALID_ARG, "recall_grad: null parameter or gradient pointer");

  // the forward GEMV keeps up to 16 x 1024 inputs in shared memory (64 KB): allow it once
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(gemv_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kGB * kCol * (int)sizeof(float));
  });
  if (attr_err != cudaSuccess) return check_cuda(attr_err, "cudaFuncSetAttribute(recall_grad)");

  const GradWs ws = carve(static_cast<float*>(workspace), B, D);
  const float* xs[3] = {h_prev, emb, h_loc};
  const size_t xsm = (size_t)B * kCol * sizeof(float);
  auto gemv = [&](const float* W, int N, int K, const float* X) {
    gemv_rows_kernel<<<dim3(N / kRowsFwd, K / kCol), 256, xsm, s>>>(W, N, K, X, K, B, ws.partA);
  };
  auto fwd = [&](FwdArgs a) {
    a.part = ws.partA;
    a.B = B;
    fwd_reduce_kernel<<<(B * a.N + 255) / 256, 256, 0, s>>>(a);
  };
  auto bwd = [&](const float* W, int N, int K, const float* dY, const float* X, float* dW, float* part) {
    const dim3 grid(N / kRowsBwd, K / kCol);
    if (B <= 8)
      bwd_rows_kernel<8><<<grid, 256, 0, s>>>(W, N, K, dY, N, X, K, B, dW, part);
    else
      bwd_rows_kernel<16><<<grid, 256, 0, s>>>(W, N, K, dY, N, X, K, B, dW, part);
  };
  auto red = [&](BwdArgs a) {
    a.B = B;
    bwd_reduce_kernel<<<B * a.K / 32, 256, 0, s>>>(a);
  };
  float* f[3] = {ws.f, ws.f + (size_t)B * kGT, ws.f + 2 * (size_t)B * kGT};

  // ---- forward recompute, keeping every activation the backward needs
  for (int i = 0; i < 3; ++i) {
    float* nx = ws.nx + (size_t)i * B * D;
    rms_kernel<<<B, 1024, 0, s>>>(xs[i], D, w->tower_norm[i], ws.sx + i * B, nx);
    gemv(w->tower_w[i], kGT, D, nx);
    FwdArgs a = {};
    a.nchunk = D / kCol;
    a.N = kGT;
    a.epi = kEpiTower;
    a.bias = w->tower_b[i];
    a.out = ws.u + (size_t)i * B * kGT;
    a.out2 = ws.p + (size_t)i * B * kGT;
    fwd(a);
  }
  interaction_kernel<<<(B * kGT + 255) / 256, 256, 0, s>>>(ws.u, B, ws.z);
  gemv(w->fuse_w, kGT, kGZ, ws.z);
  {
    FwdArgs a = {};
    a.nchunk = kGZ / kCol;
    a.N = kGT;
    a.epi = kEpiFuse;
    a.bias = w->fuse_b;
    a.u = ws.u;
    a.out = f[0];
    fwd(a);
  }
  for (int j = 0; j < 2; ++j) {
    float* m = ws.m + (size_t)j * B * kGT;
    float* g = ws.g + (size_t)j * B * kGF;
    float* v = ws.v + (size_t)j * B * kGF;
    float* act = ws.a + (size_t)j * B * kGF;
    rms_kernel<<<B, 1024, 0, s>>>(f[j], kGT, w->ffn_norm[j], ws.sf + j * B, m);
    gemv(w->ffn_gate[j], kGF, kGT, m);
    FwdArgs a = {};
    a.nchunk = 1;
    a.N = kGF;
    a.epi = kEpiStore;
    a.out = g;
    fwd(a);
    gemv(w->ffn_up[j], kGF, kGT, m);
    a.epi = kEpiUp;
    a.g = g;
    a.out = v;
    a.out2 = act;
    fwd(a);
    gemv(w->ffn_down[j], kGT, kGF, act);
    FwdArgs d = {};
    d.nchunk = kGF / kCol;
    d.N = kGT;
    d.epi = kEpiDown;
    d.f_in = f[j];
    d.out = f[j + 1];
    fwd(d);
  }
  score_kernel<<<B, 1024, 0, s>>>(f[2], w->out_norm, w->out_w, w->out_b, ws.so, ws.no, q);
  labels_kernel<<<1, 32, 0, s>>>(q, p_full, p_local, valid, B, lam, y, ws.dq, loss);

  // ---- backward
  out_grad_kernel<<<kGT / 256, 256, 0, s>>>(ws.dq, ws.no, B, gr->out_w, gr->out_b);
  norm_weight_grad_kernel<<<kGT / 256, 256, 0, s>>>(nullptr, ws.dq, w->out_w, f[2], ws.so, B, kGT,
                                                    gr->out_norm);
  rms_backward_kernel<<<B, 1024, 0, s>>>(nullptr, ws.dq, w->out_w, f[2], ws.so, w->out_norm, kGT, false,
                                        ws.dF);
  for (int j = 1; j >= 0; --j) {
    const float* m = ws.m + (size_t)j * B * kGT;
    bwd(w->ffn_down[j], kGT, kGF, ws.dF, ws.a + (size_t)j * B * kGF, gr->ffn_down[j], ws.partA);
    BwdArgs a = {};
    a.part = ws.partA;
    a.nrb = kGT / kRowsBwd;
    a.K = kGF;
    a.epi = kBwdGate;
    a.g = ws.g + (size_t)j * B * kGF;
    a.v = ws.v + (size_t)j * B * kGF;
    a.out = ws.dG;
    a.out2 = ws.dV;
    red(a);
    bwd(w->ffn_gate[j], kGF, kGT, ws.dG, m, gr->ffn_gate[j], ws.partA);
    bwd(w->ffn_up[j], kGF, kGT, ws.dV, m, gr->ffn_up[j], ws.partB);
    BwdArgs b2 = {};
    b2.part = ws.partA;
    b2.nrb = kGF / kRowsBwd;
    b2.part2 = ws.partB;
    b2.nrb2 = kGF / kRowsBwd;
    b2.K = kGT;
    b2.epi = kBwdStore;
    b2.out = ws.dM;
    red(b2);
    norm_weight_grad_kernel<<<kGT / 256, 256, 0, s>>>(ws.dM, nullptr, nullptr, f[j], ws.sf + j * B, B, kGT,
                                                      gr->ffn_norm[j]);
    rms_backward_kernel<<<B, 1024, 0, s>>>(ws.dM, nullptr, nullptr, f[j], ws.sf + j * B, w->ffn_norm[j],
                                          kGT, true, ws.dF);
  }
  batch_sum_kernel<<<kGT / 256, 256, 0, s>>>(ws.dF, B, kGT, gr->fuse_b);
  bwd(w->fuse_w, kGT, kGZ, ws.dF, ws.z, gr->fuse_w, ws.partA);
  {
    BwdArgs a = {};
    a.part = ws.partA;
    a.nrb = kGT / kRowsBwd;
    a.K = kGZ;
    a.epi = kBwdStore;
    a.out = ws.dZ;
    red(a);
  }
  fuse_backward_kernel<<<(B * kGT + 255) / 256, 256, 0, s>>>(ws.dF, ws.dZ, ws.u, ws.p, B, ws.dP);
  for (int i = 0; i < 3; ++i) {
    const float* dp = ws.dP + (size_t)i * B * kGT;
    batch_sum_kernel<<<kGT / 256, 256, 0, s>>>(dp, B, kGT, gr->tower_b[i]);
    bwd(w->tower_w[i], kGT, D, dp, ws.nx + (size_t)i * B * D, gr->tower_w[i], ws.partA);
    BwdArgs a = {};
    a.part = ws.partA;
    a.nrb = kGT / kRowsBwd;
    a.K = D;
    a.epi = kBwdStore;
    a.out = ws.dN;
    red(a);
    norm_weight_grad_kernel<<<(D + 255) / 256, 256, 0, s>>>(ws.dN, nullptr, nullptr, xs[i], ws.sx + i * B, B,
                                                            D, gr->tower_norm[i]);
  }
  return check_cuda(cudaGetLastError(), "recall_grad launch");
}

}  // namespace oda
