// Recall head R(h_{t-1}, E(x_t), h^L_t) -> q_t and the routing gate, fp32.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.2 eq. q_t and the
// paragraph after it (three inputs, per-input normalise + project + activate to 1024, a 9216-d
// interaction of the three vectors, their pairwise products and absolute differences, a
// projection with residual fusion, two residual gated feed-forward blocks, scalar output, fp32);
// §2.3 (full iff the score exceeds theta or is not finite).  Layer details follow this reading:
//   u_i = SiLU(W_i (RMSNorm(x_i) * gamma_i) + b_i)
//   f   = W_f z + b_f + (u_0 + u_1 + u_2) / 3
//   f  += W_d (SiLU(W_g m) * (W_u m)),  m = RMSNorm(f) * gamma_j      (two blocks)
//   q   = w_o . (RMSNorm(f) * gamma_o) + b_o
//
// Design: at batch sizes of a few sequences the head is a weight-streaming problem (113 MB of
// fp32 weights for D = 2048, 2*B flops per 4-byte weight) on CUDA cores.  The whole batch runs in
// one cooperative launch of all six phases (head_fused_kernel, further down), in groups of up to 8
// sequences.  Where that kernel's inputs do not fit, six phase launches run instead, each a
// split-K GEMV: a CTA streams a 32-row x Kc slab of one weight
// matrix exactly once with 16-byte non-allocating loads and multiplies it against a
// shared-memory tile of up to 8 sequences' inputs; lanes reduce with a 31-shuffle butterfly.
// The input transform of a phase (RMSNorm scale, the interaction vector, the gated activation)
// is applied while the tile is built, and the output epilogue (bias, SiLU, residual) runs in the
// last CTA of each row block, which sums the split-K partials in a fixed order (deterministic
// results).  The last row block of the final phase also computes q and the gate.  Each phase
// launch may start while the previous one finishes (programmatic dependent launch) and pulls its
// weight slab toward L2 before waiting for the previous phase's outputs.
#include <algorithm>
#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace oda {
namespace {

constexpr int kT = 1024;       // tower width
constexpr int kF = 2048;       // gated FFN width
constexpr int kHT = 256;       // threads per CTA
constexpr int kWarps = kHT / 32;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;   // 32 weight rows
constexpr int kBTMax = 8;      // sequences per tile (4 when the batch has at most 4)
constexpr float kEps = 1e-6f;

enum Phase { kTower = 0, kFuse = 1, kUp = 2, kDown = 3 };

struct HeadParams {
  oda_head_weights w;
  const float* x[3];      // h_prev, emb, h_loc  [B][D]
  const int32_t* sched;
  float* score;
  int32_t* flag;
  int32_t* any_flag;
  float* part;            // split-K partials [nchunks][B][rows_total]
  float* ss;              // tower sums of squares [row_blocks][nchunks][B]
  int32_t* cnt;           // [row blocks] + [final]
  float* u;               // [3][B][T]
  float* f;               // [3][B][T]  (f0 fusion output, f1 block 0 output, f2 block 1 output)
  float* act;             // [B][F]
  int B, D;
  int phase, block;       // block: FFN block index for kUp / kDown
  int Kc, nchunks, rows_total, row_blocks;
  float theta;
};

__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }

// Weights are read once per score when B <= 8 (streaming hint); larger batches loop over
// sequence tiles and re-read the CTA's slab, so they keep it cacheable.
__device__ __forceinline__ float4 ldg_w(const float* p, bool stream) {
  return stream ? __ldcs(reinterpret_cast<const float4*>(p))
                : __ldg(reinterpret_cast<const float4*>(p));
}

// Block-wide sums of BT per-thread values; on return red[0..BT) hold the totals (all threads
// may read them).  red must hold (kWarps + 1) * BT floats.
template <int BT>
__device__ void block_sum(float (&v)[BT], float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int bb = 0; bb < BT; ++bb)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[bb] += __shfl_xor_sync(0xffffffffu, v[bb], o);
  __syncthreads();
  if (lane == 0)
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) red[BT + warp * BT + bb] = v[bb];
  __syncthreads();
  if (threadIdx.x < BT) {
    float t = 0.f;
    for (int w = 0; w < kWarps; ++w) t += red[BT + w * BT + threadIdx.x];
    red[threadIdx.x] = t;
  }
  __syncthreads();
}

// The weight row that value slot r (0..3) of warp `warp` in row block `rb` multiplies, and
// where its partial goes (column of the partial matrix).
__device__ __forceinline__ const float* weight_row(const HeadParams& p, int rb, int warp, int r,
                                                   int* col) {
  const oda_head_weights& w = p.w;
  if (p.phase == kTower) {
    const int row = rb * kRowsPerCta + warp * kRowsPerWarp + r;   // 0 .. 3*T-1
    const int i = row / kT, n = row % kT;
    *col = row;
    return w.tower_w[i] + (size_t)n * p.D;
  }
  if (p.phase == kFuse) {
    const int n = rb * kRowsPerCta + warp * kRowsPerWarp + r;
    *col = n;
    return w.fuse_w + (size_t)n * (9 * kT);
  }
  if (p.phase == kUp) {
    // 16 FFN units per row block; a warp takes 2 units, gate rows then up rows
    const int n = rb * (kRowsPerCta / 2) + warp * 2 + (r & 1);
    const bool up = r >= 2;
    *col = (up ? kF : 0) + n;
    return (up ? w.ffn_up[p.block] : w.ffn_gate[p.block]) + (size_t)n * kT;
  }
  const int n = rb * kRowsPerCta + warp * kRowsPerWarp + r;
  *col = n;
  return w.ffn_down[p.block] + (size_t)n * kF;
}

// Four consecutive input values X[b][kg..kg+3] of a phase (kg a multiple of 4), before any
// per-sequence scaling: the tower input, the interaction vector z, f, or the gated activation.
__device__ __forceinline__ float4 tile_value4(const HeadParams& p, int rb, int b, int kg) {
  if (p.phase == kTower) {
    const int i = (rb * kRowsPerCta) / kT;
    return *reinterpret_cast<const float4*>(p.x[i] + (size_t)b * p.D + kg);
  }
  if (p.phase == kFuse) {
    const int blk = kg / kT, e = kg % kT;
    const float4 u0 = *reinterpret_cast<const float4*>(p.u + ((size_t)0 * p.B + b) * kT + e);
    const float4 u1 = *reinterpret_cast<const float4*>(p.u + ((size_t)1 * p.B + b) * kT + e);
    const float4 u2 = *reinterpret_cast<const float4*>(p.u + ((size_t)2 * p.B + b) * kT + e);
    switch (blk) {
      case 0: return u0;
      case 1: return u1;
      case 2: return u2;
      case 3: return make_float4(u0.x * u1.x, u0.y * u1.y, u0.z * u1.z, u0.w * u1.w);
      case 4: return make_float4(u0.x * u2.x, u0.y * u2.y, u0.z * u2.z, u0.w * u2.w);
      case 5: return make_float4(u1.x * u2.x, u1.y * u2.y, u1.z * u2.z, u1.w * u2.w);
      case 6: return make_float4(fabsf(u0.x - u1.x), fabsf(u0.y - u1.y), fabsf(u0.z - u1.z), fabsf(u0.w - u1.w));
      case 7: return make_float4(fabsf(u0.x - u2.x), fabsf(u0.y - u2.y), fabsf(u0.z - u2.z), fabsf(u0.w - u2.w));
      default: return make_float4(fabsf(u1.x - u2.x), fabsf(u1.y - u2.y), fabsf(u1.z - u2.z), fabsf(u1.w - u2.w));
    }
  }
  if (p.phase == kUp)   // scaled by the RMSNorm below
    return *reinterpret_cast<const float4*>(p.f + ((size_t)p.block * p.B + b) * kT + kg);
  return *reinterpret_cast<const float4*>(p.act + (size_t)b * kF + kg);
}

// Builds the input tile X[bb][0..Kc) for sequences b0..b0+BT-1 of chunk `chunk` (zeros beyond B).
// 16-byte loads, four per thread in flight before any is stored.
template <int BT>
__device__ void build_tile(const HeadParams& p, int rb, int chunk, int b0, float* X, float* ss_out,
                           float* red) {
  const int k0 = chunk * p.Kc;
  const int kc4 = p.Kc / 4, n4 = BT * kc4;
  float4* X4 = reinterpret_cast<float4*>(X);
  for (int base = threadIdx.x; base < n4; base += 4 * kHT) {
    float4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int idx = base + j * kHT;
      v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (idx < n4) {
        const int bb = idx / kc4, k4 = idx - bb * kc4;
        if (b0 + bb < p.B) v[j] = tile_value4(p, rb, b0 + bb, k0 + 4 * k4);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (base + j * kHT < n4) X4[base + j * kHT] = v[j];
  }
  __syncthreads();
  if (p.phase == kTower) {
    // sums of squares of this chunk of x_i for the BT sequences of the tile, one pass
    const int i = (rb * kRowsPerCta) / kT;
    float ssq[BT];
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) {
      ssq[bb] = 0.f;
      for (int k = threadIdx.x; k < p.Kc; k += kHT) ssq[bb] += X[bb * p.Kc + k] * X[bb * p.Kc + k];
    }
    block_sum<BT>(ssq, red);
    if (threadIdx.x < BT && b0 + threadIdx.x < p.B)
      ss_out[((size_t)rb * p.nchunks + chunk) * p.B + b0 + threadIdx.x] = red[threadIdx.x];
    const float* gam = p.w.tower_norm[i] + k0;
    for (int idx = threadIdx.x; idx < BT * p.Kc; idx += kHT) X[idx] *= gam[idx % p.Kc];
    __syncthreads();
  } else if (p.phase == kUp) {
    // m = RMSNorm(f) * gamma over the full 1024-wide f, one pass for the BT sequences (from the
    // tile itself when it holds the whole of f)
    const float* gam = p.w.ffn_norm[p.block] + k0;
    float ssq[BT];
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) {
      ssq[bb] = 0.f;
      if (b0 + bb < p.B) {
        const float* fr = p.Kc == kT ? X + bb * kT : p.f + ((size_t)p.block * p.B + b0 + bb) * kT;
        for (int k = threadIdx.x; k < kT; k += kHT) ssq[bb] += fr[k] * fr[k];
      }
    }
    block_sum<BT>(ssq, red);
    for (int idx = threadIdx.x; idx < BT * p.Kc; idx += kHT) {
      const int bb = idx / p.Kc, k = idx % p.Kc;
      X[idx] *= rsqrtf(red[bb] / kT + kEps) * gam[k];
    }
    __syncthreads();
  }
}

// q = w_o . (RMSNorm(f2) * gamma_o) + b_o for sequence b (whole warp; f2 row written by other
// CTAs of this launch or an earlier one) and its gate: full iff q > theta or q is not finite,
// or the scheduled flag where a schedule is given.
__device__ __forceinline__ void score_and_gate(const oda_head_weights& w, const float* fr, int b,
                                               const int32_t* sched, float theta, float* score,
                                               int32_t* flag, int* s_any, int lane) {
  float ss = 0.f, dot = 0.f;
  for (int k = lane; k < kT; k += 32) {
    const float fv = __ldcg(fr + k);
    ss += fv * fv;
    dot += w.out_w[k] * w.out_norm[k] * fv;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  if (lane == 0) {
    const float q = dot * rsqrtf(ss / kT + kEps) + w.out_b[0];
    score[b] = q;
    int fl;
    if (sched) {
      fl = sched[b] != 0;
    } else {
      const bool nonfinite = (__float_as_uint(q) & 0x7f800000u) == 0x7f800000u;
      fl = (nonfinite || q > theta) ? 1 : 0;
    }
    flag[b] = fl;
    if (fl) atomicOr(s_any, 1);
  }
}

// Split-K partials of output column `col` for sequence b, summed in chunk order; all loads are
// issued before the first add (at most kMaxChunks chunks).
constexpr int kMaxChunks = 16;
__device__ __forceinline__ float sum_chunks(const HeadParams& p, int b, int col) {
  float v[kMaxChunks];
#pragma unroll
  for (int ch = 0; ch < kMaxChunks; ++ch)
    v[ch] = ch < p.nchunks ? __ldcg(p.part + ((size_t)ch * p.B + b) * p.rows_total + col) : 0.f;
  float acc = 0.f;
#pragma unroll
  for (int ch = 0; ch < kMaxChunks; ++ch) acc += v[ch];
  return acc;
}

// BT: sequences per tile (4 or 8); NB: register buffers of weights (NB rounds of 32 lanes x 4
// rows x 16 bytes in flight per warp), 4 with 4-wide tiles and 2 with 8-wide ones, so both fit
// the same 128 registers.
template <int BT, int NB>
__global__ void __launch_bounds__(kHT) head_phase_kernel(const HeadParams p) {
  extern __shared__ float X[];           // [BT][Kc]
  __shared__ float red[BT + kWarps * BT];
  __shared__ int s_last;
  const int rb = blockIdx.x / p.nchunks, chunk = blockIdx.x % p.nchunks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = chunk * p.Kc;

  int cols[kRowsPerWarp];
  const float* wrow[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) wrow[r] = weight_row(p, rb, warp, r, &cols[r]) + k0;
  // The weights never change: pull this CTA's slab toward L2 and load its first NB rounds into
  // registers while the previous phase may still be running (programmatic dependent launch),
  // then wait for its outputs.
  const bool single_pass = p.B <= BT;
  const int n4 = p.Kc / 4;   // >= 64 in every phase
  float4 wbuf[NB][kRowsPerWarp];
  auto load_w = [&](float4 (&w)[kRowsPerWarp], int k4) {
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) w[r] = ldg_w(wrow[r] + 4 * k4, single_pass);
  };
  auto load_first = [&]() {
#pragma unroll
    for (int j = 0; j < NB; ++j)
      if (lane + 32 * j < n4) load_w(wbuf[j], lane + 32 * j);
  };
  for (int r = 0; r < kRowsPerWarp; ++r)
    for (int k = lane * 32 + 128 * NB; k < p.Kc; k += 32 * 32)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow[r] + k));
  load_first();
  grid_dependency_wait();
  grid_dependents_launch();

  for (int b0 = 0; b0 < p.B; b0 += BT) {
    if (b0 > 0) load_first();   // later sequence tiles read the slab again
    build_tile<BT>(p, rb, chunk, b0, X, p.ss, red);
    float acc[kRowsPerWarp][BT];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) acc[r][bb] = 0.f;
    auto fma_w = [&](const float4 (&w)[kRowsPerWarp], int k4) {
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) {
        const float4 xv = *reinterpret_cast<const float4*>(X + bb * p.Kc + 4 * k4);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
          acc[r][bb] += w[r].x * xv.x + w[r].y * xv.y + w[r].z * xv.z + w[r].w * xv.w;
      }
    };
    // NB register buffers, each refilled NB rounds ahead of its use
    for (int k4 = lane; k4 < n4; k4 += 32 * NB) {
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const int kk = k4 + 32 * j;
        if (kk < n4) {
          fma_w(wbuf[j], kk);
          if (kk + 32 * NB < n4) load_w(wbuf[j], kk + 32 * NB);
        }
      }
    }
    // butterfly over the kRowsPerWarp * BT values (32 or 16): afterwards lane l holds the
    // lane-sum of value l % NV (r = (l % NV) / BT, bb = l % BT)
    constexpr int NV = kRowsPerWarp * BT;
    float v[NV];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) v[r * BT + bb] = acc[r][bb];
#pragma unroll
    for (int half = NV / 2; half >= 1; half >>= 1) {
      const bool upper = (lane & half) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
      }
    }
#pragma unroll
    for (int o = NV; o < 32; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    if (p.phase == kUp && p.nchunks == 1) {
      // whole rows: lanes [0, 2 BT) hold the gate sums of the warp's two units, lanes
      // [2 BT, 4 BT) the up sums of the same units; act = SiLU(gate) * up
      const float up = __shfl_down_sync(0xffffffffu, v[0], 2 * BT);
      const int r = lane / BT, bb = lane % BT, b = b0 + bb;
      if (lane < 2 * BT && b < p.B) {
        const int n = rb * (kRowsPerCta / 2) + warp * 2 + r;
        p.act[(size_t)b * kF + n] = silu(v[0]) * up;
      }
    } else if (lane < NV) {
      const int r = lane / BT, bb = lane % BT, b = b0 + bb;
      int col = cols[0];
#pragma unroll
      for (int rr = 1; rr < kRowsPerWarp; ++rr)
        if (r == rr) col = cols[rr];
      if (b < p.B) p.part[((size_t)chunk * p.B + b) * p.rows_total + col] = v[0];
    }
    __syncthreads();
  }

  // ---- last CTA of the row block: reduce partials in chunk order and apply the epilogue
  // (the up projection over whole rows has written its output already)
  if (p.phase == kUp && p.nchunks == 1) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&p.cnt[rb], 1) == p.nchunks - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int units = (p.phase == kUp) ? kRowsPerCta / 2 : kRowsPerCta;
  for (int idx = threadIdx.x; idx < units * p.B; idx += kHT) {
    const int j = idx % units, b = idx / units;
    if (p.phase == kTower) {
      const int row = rb * kRowsPerCta + j, i = row / kT, n = row % kT;
      const float acc = sum_chunks(p, b, row);
      float ss = 0.f;
      for (int ch = 0; ch < p.nchunks; ++ch) ss += __ldcg(p.ss + ((size_t)rb * p.nchunks + ch) * p.B + b);
      const float inv = rsqrtf(ss / p.D + kEps);
      p.u[((size_t)i * p.B + b) * kT + n] = silu(acc * inv + p.w.tower_b[i][n]);
    } else if (p.phase == kFuse) {
      const int n = rb * kRowsPerCta + j;
      const float acc = sum_chunks(p, b, n);
      const float mean = (__ldcg(p.u + ((size_t)0 * p.B + b) * kT + n) +
                          __ldcg(p.u + ((size_t)1 * p.B + b) * kT + n) +
                          __ldcg(p.u + ((size_t)2 * p.B + b) * kT + n)) / 3.0f;
      p.f[((size_t)0 * p.B + b) * kT + n] = acc + p.w.fuse_b[n] + mean;
    } else if (p.phase == kUp) {
      const int n = rb * (kRowsPerCta / 2) + j;
      const float ga = sum_chunks(p, b, n), ua = sum_chunks(p, b, kF + n);
      p.act[(size_t)b * kF + n] = silu(ga) * ua;
    } else {
      const int n = rb * kRowsPerCta + j;
      const float acc = sum_chunks(p, b, n);
      p.f[((size_t)(p.block + 1) * p.B + b) * kT + n] =
          __ldcg(p.f + ((size_t)p.block * p.B + b) * kT + n) + acc;
    }
  }
  if (threadIdx.x == 0) p.cnt[rb] = 0;
  if (!(p.phase == kDown && p.block == 1)) return;

  // ---- final row block done: q = w_o . (RMSNorm(f2) * gamma_o) + b_o and the gate
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&p.cnt[p.row_blocks], 1) == p.row_blocks - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  __shared__ int s_any;
  if (threadIdx.x == 0) s_any = 0;
  __syncthreads();
  for (int b = warp; b < p.B; b += kWarps)
    score_and_gate(p.w, p.f + ((size_t)2 * p.B + b) * kT, b, p.sched, p.theta, p.score, p.flag,
                   &s_any, lane);
  __syncthreads();
  if (threadIdx.x == 0) {
    *p.any_flag = s_any;
    p.cnt[p.row_blocks] = 0;
  }
}

// ------------------------------------------------------------ fused head
// One cooperative launch, one CTA per SM, runs all six phases.  The batch is cut into groups of
// up to 8 sequences (the tile width), each on its own share of the grid; every group streams all
// the weights, and as CTA i of each group reads the same segments in the same order, in step with
// the other groups through the phase barriers, HBM serves a segment once and L2 the other groups.
// Warp 8 streams every weight row segment (1024 floats, 4 KiB) the CTA owns through a ring of
// 32 KiB stages with bulk copies,
// phase after phase: the weights never depend on a phase's inputs, so HBM keeps streaming while
// the grid waits between phases.  Warps 0-7 take one segment each per stage and dot it against
// the phase's input, held whole in shared memory for the sequence tile.  Each CTA owns whole
// output rows of every phase (all of their K-chunks), so it finishes them itself (norm scale,
// bias, activation, residual) and no split-K partial leaves the SM; a grid-wide barrier (a
// counter with a bounded spin) separates the phases.  The last CTA to finish computes q and the
// gate.
constexpr int kFC = 8;                              // consumer warps
constexpr int kFThreads = (kFC + 1) * 32;           // + one producer warp
constexpr int kSeg = 1024;                          // floats per weight segment
constexpr int kSegBytes = kSeg * 4;
constexpr int kFStageBytes = kFC * kSegBytes;       // one segment per consumer warp
constexpr int kMaxRing = 5;
constexpr int kMaxOwnSegs = 32;                     // segments of one batch of a CTA's rows
constexpr uint64_t kFWaitNs = 2000000000ull;
constexpr uint64_t kGridWaitNs = 1000000000ull;

struct FusedParams {
  oda_head_weights w;
  const float* x[3];      // h_prev, emb, h_loc  [B][D]
  const int32_t* sched;
  float* score;
  int32_t* flag;
  int32_t* any_flag;
  float* u;               // [3][B][T]
  float* f;               // [3][B][T]
  float* act;             // [B][F]
  int32_t* cnt;           // [0] grid-barrier arrivals, [1] finished CTAs; both back to 0 at exit
  int32_t* err;
  int B, D, ring;
  int groups, gsize;      // sequence groups of the tile width, and CTAs per group
  float theta;
};

// The rows of phase ph (0 tower, 1 fuse, 2 up 0, 3 down 0, 4 up 1, 5 down 1) that CTA c of G
// owns: [lo, lo + n) (gate/up row pairs for the up projections); the tower phase splits the
// grid into three groups, one per tower.  nseg: weight segments per K-chunk.
struct Own {
  int kind, blk, tower, lo, n, nchunk, nseg;
};

__device__ __forceinline__ Own own_rows(int ph, int c, int G, int D) {
  Own o;
  o.kind = ph == 0 ? kTower : ph == 1 ? kFuse : ((ph & 1) == 0 ? kUp : kDown);
  o.blk = ph >= 4 ? 1 : 0;
  o.tower = 0;
  int rows = kT, cc = c, gg = G;
  if (o.kind == kTower) {
    int i = 0;
    while (i < 2 && (long long)G * (i + 1) / 3 <= c) ++i;
    const int g0 = (int)((long long)G * i / 3), g1 = (int)((long long)G * (i + 1) / 3);
    o.tower = i;
    cc = c - g0;
    gg = g1 - g0;
  } else if (o.kind == kUp) {
    rows = kF;
  }
  o.lo = (int)((long long)rows * cc / gg);
  o.n = (int)((long long)rows * (cc + 1) / gg) - o.lo;
  o.nchunk = o.kind == kTower ? D / kSeg : o.kind == kFuse ? 9 : o.kind == kUp ? 1 : kF / kSeg;
  o.nseg = o.kind == kUp ? 2 * o.n : o.n;
  return o;
}

// A CTA takes its rows of a phase in batches of at most kMaxOwnSegs segments (gate/up rows of the
// same units stay together), the size of its row-sum area.  With one sequence group every CTA
// owns few enough rows for one batch; with several groups each CTA owns more rows.
__device__ __forceinline__ int batch_rows(const Own& o) { return o.kind == kUp ? kMaxOwnSegs / 2 : kMaxOwnSegs; }
__device__ __forceinline__ int n_batches(const Own& o) { return (o.n + batch_rows(o) - 1) / batch_rows(o); }
__device__ __forceinline__ Own batch_of(Own o, int j) {
  const int per = batch_rows(o);
  o.lo += j * per;
  o.n = min(per, o.n - j * per);
  o.nseg = o.kind == kUp ? 2 * o.n : o.n;
  return o;
}

// Segment r of K-chunk ch of the CTA's rows (for the up projections r < n are gate rows and
// r >= n the up rows of the same units).
__device__ __forceinline__ const float* seg_ptr(const FusedParams& p, const Own& o, int ch, int r) {
  const oda_head_weights& w = p.w;
  switch (o.kind) {
    case kTower: return w.tower_w[o.tower] + (size_t)(o.lo + r) * p.D + ch * kSeg;
    case kFuse: return w.fuse_w + (size_t)(o.lo + r) * (9 * kT) + ch * kSeg;
    case kUp:
      return r < o.n ? w.ffn_gate[o.blk] + (size_t)(o.lo + r) * kT
                     : w.ffn_up[o.blk] + (size_t)(o.lo + r - o.n) * kT;
    default: return w.ffn_down[o.blk] + (size_t)(o.lo + r) * kF + ch * kSeg;
  }
}

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kFC * 32) : "memory");
}

// Butterfly over 32 values: afterwards lane l holds the sum over the warp of value l.
__device__ __forceinline__ float butterfly32(float (&v)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}


// This warp's 128-column slice of K-chunk ch of the phase input, lane l holding columns
// 4*col4 .. 4*col4+3 of the chunk, for the BT sequences of the tile (zeros beyond B).  Tower:
// the raw x_i rows are in `src` ([B][D]); the slice is x*gamma and ssl collects x^2.  Fuse: z is
// formed from u_0, u_1, u_2 ([3][BT][T]): chunk 0-2 is u_c, 3-5 the products u0u1, u0u2, u1u2,
// 6-8 the absolute differences in the same order.
template <int BT>
__device__ __forceinline__ void input_slice(const Own& o, int B, int D, const float* src, int ch,
                                            int col4, float4 gam, float (&ssl)[BT], float4 (&xs)[BT]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  if (o.kind == kTower) {
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) {
      const float4 x = bb < B ? s4[(size_t)bb * (D / 4) + ch * (kSeg / 4) + col4] : zero;
      ssl[bb] += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
      xs[bb] = make_float4(x.x * gam.x, x.y * gam.y, x.z * gam.z, x.w * gam.w);
    }
  } else if (o.kind == kFuse) {
    const int m = (ch + 6) % 3;   // 0, 1, 2 for chunks 3|6, 4|7, 5|8
    const int ia = ch < 3 ? ch : (m == 2 ? 1 : 0), ib = ch < 3 ? ch : (m == 0 ? 1 : 2);
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) {
      const float4 a = s4[(ia * BT + bb) * (kT / 4) + col4];
      if (ch < 3) {
        xs[bb] = a;
      } else {
        const float4 b = s4[(ib * BT + bb) * (kT / 4) + col4];
        xs[bb] = ch < 6 ? make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w)
                        : make_float4(fabsf(a.x - b.x), fabsf(a.y - b.y), fabsf(a.z - b.z),
                                      fabsf(a.w - b.w));
      }
    }
  } else if (o.kind == kUp) {
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) xs[bb] = s4[bb * (kT / 4) + col4];
  } else {
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) xs[bb] = s4[bb * (kF / 4) + ch * (kSeg / 4) + col4];
  }
}

// The warp's share of one stage: its 128 columns of each of the n (<= 8) segments, dotted with
// the input slice; 32 values per butterfly (segments x sequences), and the lane holding value
// (segment i, sequence bb) adds it to the warp's row sum acc[(8g + i)][bb].
template <int BT>
__device__ __forceinline__ void stage_dot(const uint8_t* stage, int n, int col4, const float4 (&xs)[BT],
                                          float* acc, int g, int lane) {
  constexpr int NS = 32 / BT;   // segments per butterfly
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int hf = 0; hf < kFC / NS; ++hf) {
    float v[32];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const int si = hf * NS + i;
      const float4 w = si < n ? reinterpret_cast<const float4*>(stage + si * kSegBytes)[col4] : zero;
#pragma unroll
      for (int bb = 0; bb < BT; ++bb)
        v[i * BT + bb] = w.x * xs[bb].x + w.y * xs[bb].y + w.z * xs[bb].z + w.w * xs[bb].w;
    }
    const float t = butterfly32(v, lane);
    const int si = hf * NS + lane / BT;
    if (si < n) acc[(g * kFC + si) * BT + lane % BT] += t;
  }
}

// The input of the fuse, up and down phases for the sequence tile, into shared memory (zeros
// beyond B): fuse u_0, u_1, u_2 [3][BT][T]; up f_j * gamma_j [BT][T] (inv[bb] receives 1 / rms(f_j),
// applied to the dot products); down act [BT][F].  These rows were written by other CTAs of
// this launch (L2 loads).  Ends with a consumer barrier.
template <int BT>
__device__ void load_source(const FusedParams& p, const Own& o, int b0, int Bs, float* src, float* red,
                            float* inv, int tid) {
  const int B = p.B, lane = tid & 31, warp = tid >> 5;
  float4* s4 = reinterpret_cast<float4*>(src);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  if (o.kind == kUp) {
    float ss[BT];
    const float4* g4 = reinterpret_cast<const float4*>(p.w.ffn_norm[o.blk]);
    float4 v[BT];   // kT / 4 == 256 == consumer threads: one float4 of f per sequence each
#pragma unroll
    for (int bb = 0; bb < BT; ++bb)
      v[bb] = bb < Bs ? __ldcg(reinterpret_cast<const float4*>(p.f + ((size_t)o.blk * B + b0 + bb) * kT) + tid) : zero;
    const float4 g = g4[tid];
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) {
      ss[bb] = v[bb].x * v[bb].x + v[bb].y * v[bb].y + v[bb].z * v[bb].z + v[bb].w * v[bb].w;
      s4[bb * (kT / 4) + tid] = make_float4(v[bb].x * g.x, v[bb].y * g.y, v[bb].z * g.z, v[bb].w * g.w);
    }
#pragma unroll
    for (int bb = 0; bb < BT; ++bb)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss[bb] += __shfl_xor_sync(0xffffffffu, ss[bb], off);
    if (lane == 0)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) red[warp * BT + bb] = ss[bb];
    consumer_sync();
    if (tid < BT) {
      float t = 0.f;
      for (int w = 0; w < kFC; ++w) t += red[w * BT + tid];
      inv[tid] = rsqrtf(t / kT + kEps);
    }
  } else if (o.kind == kFuse) {
    // every load is issued before the first store
    float4 v[3][BT];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb)
        v[i][bb] = bb < Bs ? __ldcg(reinterpret_cast<const float4*>(p.u + ((size_t)i * B + b0 + bb) * kT) + tid)
                           : zero;
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) s4[(i * BT + bb) * (kT / 4) + tid] = v[i][bb];
  } else {
    float4 v[BT][2];
#pragma unroll
    for (int bb = 0; bb < BT; ++bb)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        v[bb][j] = bb < Bs ? __ldcg(reinterpret_cast<const float4*>(p.act + (size_t)(b0 + bb) * kF) + tid + j * kFC * 32)
                           : zero;
#pragma unroll
    for (int bb = 0; bb < BT; ++bb)
#pragma unroll
      for (int j = 0; j < 2; ++j) s4[bb * (kF / 4) + tid + j * kFC * 32] = v[bb][j];
  }
  consumer_sync();
}

// The operand of output item idx (row idx / Bs, sequence b0 + idx % Bs) of the phase that comes
// from global memory: the tower or fusion bias, or the residual f_j of a down projection (written
// two phases earlier).  Each thread loads the one for its own item while the phase's stages stream.
__device__ __forceinline__ float finish_operand(const FusedParams& p, const Own& o, int b0, int Bs, int idx) {
  if (idx >= o.n * Bs) return 0.f;
  const int r = idx / Bs, b = idx - r * Bs, n = o.lo + r;
  switch (o.kind) {
    case kTower: return p.w.tower_b[o.tower][n];
    case kFuse: return p.w.fuse_b[n];
    case kUp: return 0.f;
    default: return __ldcg(p.f + ((size_t)o.blk * p.B + b0 + b) * kT + n);
  }
}

// Finishes the CTA's rows of the phase; the dot product of row segment r for sequence b is the
// sum of the eight warps' column shares accw[w][r][b], taken in warp order.  `pre` is this
// thread's finish_operand.
template <int BT>
__device__ void finish_rows(const FusedParams& p, const Own& o, int b0, int Bs, const float* src,
                            const float* accw, const float* inv, float pre, int tid) {
  const int B = p.B;
  auto rowsum = [&](int r, int b) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kFC; ++w) t += accw[(w * kMaxOwnSegs + r) * BT + b];
    return t;
  };
  for (int idx = tid; idx < o.n * Bs; idx += kFC * 32) {
    const int r = idx / Bs, b = idx - r * Bs, n = o.lo + r;
    const float acc = rowsum(r, b);
    const float opnd = idx == tid ? pre : finish_operand(p, o, b0, Bs, idx);
    if (o.kind == kTower) {
      p.u[((size_t)o.tower * B + b0 + b) * kT + n] = silu(acc * inv[b] + opnd);
    } else if (o.kind == kFuse) {
      const float mean = (src[(0 * BT + b) * kT + n] + src[(1 * BT + b) * kT + n] +
                          src[(2 * BT + b) * kT + n]) / 3.0f;
      p.f[(size_t)(b0 + b) * kT + n] = acc + opnd + mean;
    } else if (o.kind == kUp) {
      const float ga = acc * inv[b], ua = rowsum(o.n + r, b) * inv[b];
      p.act[(size_t)(b0 + b) * kF + n] = silu(ga) * ua;
    } else {
      p.f[((size_t)(o.blk + 1) * B + b0 + b) * kT + n] = opnd + acc;
    }
  }
}

// kGroups: the batch is cut into sequence groups on shares of the grid (batches above the tile
// width); without it one group spans the grid and every CTA's rows of a phase fit one batch
// (at least 128 SMs), so that instantiation carries neither the group offsets nor the batch loop.
template <int BT, bool kGroups>
__global__ void __launch_bounds__(kFThreads, 1) head_fused_kernel(const FusedParams p) {
  extern __shared__ __align__(16) uint8_t fsm[];
  const int R = p.ring;
  uint8_t* ring = fsm;
  float* src = reinterpret_cast<float*>(fsm + (size_t)R * kFStageBytes);
  float* accw = src + (size_t)max(p.D, 3 * kT) * BT;     // [kFC][kMaxOwnSegs][BT]
  __shared__ __align__(8) uint64_t full[kMaxRing];
  __shared__ __align__(8) uint64_t empty[kMaxRing];
  __shared__ __align__(8) uint64_t src_bar;
  __shared__ float red[kFC * BT];
  __shared__ float s_inv[BT];
  __shared__ int s_last, s_any;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = gridDim.x, B = p.B;
  // sequence group of this CTA: sequences [b0, b0 + Bs) on CTAs [grp * gsize, grp * gsize + gsize);
  // CTAs past the last group own no rows and only take part in the grid barriers
  const int grp = kGroups ? c / p.gsize : 0;
  const int cg = kGroups ? c - grp * p.gsize : c;
  const int b0 = kGroups ? grp * BT : 0;
  const int Bs = kGroups ? (grp < p.groups ? min(BT, B - b0) : 0) : B;
  auto own = [&](int ph) {
    Own o = own_rows(ph, cg, kGroups ? p.gsize : G, p.D);
    if (kGroups && Bs == 0) o.n = o.nseg = 0;
    return o;
  };
  auto nbatches = [&](const Own& o) { return kGroups ? n_batches(o) : 1; };
  auto batch = [&](const Own& o, int j) { return kGroups ? batch_of(o, j) : o; };
  if (tid == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kFC);
    }
    mbar_init(&src_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kFC) {
    // ---- producer.  First the tower input rows x_i[b] of this CTA's tower and sequence group
    // (they may come from the previous kernel), then every weight segment of every phase in the
    // order the consumers take them, running up to the ring's depth ahead of them (into the next
    // phase while they finish one or wait at a barrier).  No L2 prefetch ahead of the ring: the
    // copy engine takes requests in order, so bulk prefetches delay the ring's own copies (with L2
    // flushed between scores, 55.5 us per score with them, 51.5 without), and line prefetches
    // issued at the phase boundaries compete with the copies in flight (61.8 vs 55.7 us).
    grid_dependency_wait();
    const Own o0 = own(0);
    if (lane == 0) mbar_arrive_expect_tx(&src_bar, (uint32_t)(Bs * p.D * sizeof(float)));
    __syncwarp();
    if (lane < Bs)
      bulk_load(src + (size_t)lane * p.D, p.x[o0.tower] + (size_t)(b0 + lane) * p.D,
                (uint32_t)(p.D * sizeof(float)), &src_bar);
    int k = 0;
    for (int ph = 0; ph < 6; ++ph) {
      const Own oa = own(ph);
      const int nbat = nbatches(oa);
      for (int j = 0; j < nbat; ++j) {
        const Own o = batch(oa, j);
        const int ngrp = (o.nseg + kFC - 1) / kFC;
        for (int ch = 0; ch < o.nchunk; ++ch)
          for (int g = 0; g < ngrp; ++g, ++k) {
            const int s = k % R;
            if (k >= R && !mbar_wait_bounded(&empty[s], (uint32_t)(k / R - 1) & 1u, kFWaitNs) && lane == 0)
              atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
            const int n = min(kFC, o.nseg - g * kFC);
            if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(n * kSegBytes));
            __syncwarp();
            if (lane < n)
              bulk_load(ring + (size_t)s * kFStageBytes + lane * kSegBytes, seg_ptr(p, o, ch, g * kFC + lane),
                        kSegBytes, &full[s]);
          }
      }
    }
    return;
  }

  // ---- consumers: warp w owns columns [128w, 128w + 128) of every segment
  grid_dependency_wait();
  grid_dependents_launch();
  float* acc = accw + (size_t)warp * kMaxOwnSegs * BT;
  const int col4 = 32 * warp + lane;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  int k = 0;
  for (int ph = 0; ph < 6; ++ph) {
    const Own oa = own(ph);
    const bool tower = oa.kind == kTower;
    const float4* gam4 = reinterpret_cast<const float4*>(p.w.tower_norm[oa.tower]);
    // one group: the tower norm weights of the first chunk, loaded before the input wait
    const float4 gfirst = !kGroups && tower ? __ldg(gam4 + col4) : zero;
    if (tower) {
      if (!mbar_wait_bounded(&src_bar, 0u, kFWaitNs) && lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
    } else {
      load_source<BT>(p, oa, b0, Bs, src, red, s_inv, tid);
    }
    const int nbat = nbatches(oa);
    for (int j = 0; j < nbat; ++j) {
      const Own o = batch(oa, j);
      for (int i = lane; i < kMaxOwnSegs * BT; i += 32) acc[i] = 0.f;
      float4 gnext = kGroups ? (tower ? __ldg(gam4 + col4) : zero) : gfirst;
      __syncwarp();
      const float pre = finish_operand(p, o, b0, Bs, tid);
      float ssl[BT];
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) ssl[bb] = 0.f;
      const int ngrp = (o.nseg + kFC - 1) / kFC;
      for (int ch = 0; ch < o.nchunk; ++ch) {
        const float4 gam = gnext;
        if (tower && ch + 1 < o.nchunk) gnext = __ldg(gam4 + (ch + 1) * (kSeg / 4) + col4);
        float4 xs[BT];
        input_slice<BT>(o, Bs, p.D, src, ch, col4, gam, ssl, xs);
        for (int g = 0; g < ngrp; ++g, ++k) {
          const int s = k % R;
          if (!mbar_wait_bounded(&full[s], (uint32_t)(k / R) & 1u, kFWaitNs) && lane == 0)
            atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
          stage_dot<BT>(ring + (size_t)s * kFStageBytes, min(kFC, o.nseg - g * kFC), col4, xs, acc, g, lane);
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
      }
      if (tower) {
        // 1 / rms(x_i): the warps' column shares of the sum of squares, summed in warp order (the
        // same value for every batch of rows)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb)
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) ssl[bb] += __shfl_xor_sync(0xffffffffu, ssl[bb], off);
        if (lane == 0)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) red[warp * BT + bb] = ssl[bb];
        consumer_sync();
        if (tid < BT) {
          float t = 0.f;
          for (int w = 0; w < kFC; ++w) t += red[w * BT + tid];
          s_inv[tid] = rsqrtf(t / p.D + kEps);
        }
      }
      consumer_sync();
      finish_rows<BT>(p, o, b0, Bs, src, accw, s_inv, pre, tid);
      consumer_sync();
    }
    if (ph < 5) {
      if (tid == 0 && !grid_barrier_bounded(p.cnt, (ph + 1) * G, kGridWaitNs)) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
      consumer_sync();
    }
  }

  // ---- the last CTA to finish computes q and the gate of every sequence, then returns the
  // counters to zero
  if (tid == 0) {
    s_last = atom_add_acq_rel_gpu(p.cnt + 1, 1) == G - 1;
    s_any = 0;
  }
  consumer_sync();
  if (!s_last) return;
  for (int b = warp; b < B; b += kFC)
    score_and_gate(p.w, p.f + ((size_t)2 * B + b) * kT, b, p.sched, p.theta, p.score, p.flag,
                   &s_any, lane);
  consumer_sync();
  if (tid == 0) {
    *p.any_flag = s_any;
    p.cnt[0] = 0;
    p.cnt[1] = 0;
  }
}

struct PhaseShape {
  int Kc, nchunks, rows_total, row_blocks;
};

PhaseShape phase_shape(int phase, int D) {
  switch (phase) {
    case kTower: return {D / 2, 2, 3 * kT, 3 * kT / kRowsPerCta};
    case kFuse: return {1024, 9, kT, kT / kRowsPerCta};
    case kUp: return {kT, 1, 2 * kF, kF / (kRowsPerCta / 2)};   // whole rows: epilogue in registers
    default: return {256, kF / 256, kT, kT / kRowsPerCta};
  }
}

}  // namespace

size_t head_part_floats(int B, int D) {
  size_t m = 0;
  for (int ph = 0; ph < 4; ++ph) {
    const PhaseShape s = phase_shape(ph, D);
    m = std::max(m, (size_t)s.nchunks * B * s.rows_total);
  }
  return m;
}

// Per-chunk sums of squares of the tower inputs: (row block, chunk, sequence) of the tower phase.
size_t head_ss_floats(int B, int D) {
  const PhaseShape s = phase_shape(kTower, D);
  return (size_t)s.row_blocks * s.nchunks * B;
}

int head_counter_count(int D) {
  int m = 0;
  for (int ph = 0; ph < 4; ++ph) m = std::max(m, phase_shape(ph, D).row_blocks);
  return m + 1;
}

namespace {
// device properties and the fused kernels' static shared memory, read by prepare_head_kernel
int g_fused_static[3] = {-1, -1, -1};   // head_fused_kernel<4, false>, <8, false>, <8, true>

// The fused kernel for a plan's tile width and grouping, and its index above.
using FusedKernel = void (*)(FusedParams);
int fused_index(int bt, bool grouped) { return bt == 4 ? 0 : grouped ? 2 : 1; }
FusedKernel fused_kernel(int index) {
  return index == 0 ? head_fused_kernel<4, false> : index == 1 ? head_fused_kernel<8, false>
                                                                : head_fused_kernel<8, true>;
}
int g_smem_optin = 0;
int g_coop = 0;

// Fused-head plan: sequence tile, sequence groups, ring depth and dynamic shared memory; bt = 0
// where the fused kernel does not apply (D not a multiple of 1024, fewer than 128 SMs, no
// cooperative launch, or too little shared memory for a ring of two stages), and the six phase
// kernels run instead.
struct FusedPlan {
  int bt, groups, gsize, ring;
  bool grouped;   // the kernel with sequence groups and row batches
  size_t smem;
};

FusedPlan fused_plan(int B, int D, int n_sms) {
  FusedPlan pl = {0, 0, 0, 0, false, 0};
  if (B < 1 || D % kSeg != 0 || n_sms < 128 || !g_coop) return pl;
  const int bt = B <= 4 ? 4 : 8;
  const int groups = (B + bt - 1) / bt;
  const int gsize = n_sms / groups;
  if (gsize < 3) return pl;   // the tower phase gives each of the three towers a CTA at least
  // one group whose CTAs each own few enough rows of every phase for one batch (true from about
  // 96 SMs) runs the kernel without groups and batches; a 4-wide tile never needs them
  const int g3 = gsize / 3;
  const bool one_batch = (kT + g3 - 1) / g3 <= kMaxOwnSegs && (kF + gsize - 1) / gsize <= kMaxOwnSegs / 2;
  const bool grouped = groups > 1 || !one_batch;
  if (grouped && bt == 4) return pl;
  const int stat = g_fused_static[fused_index(bt, grouped)];
  if (stat < 0) return pl;
  const size_t src = (size_t)std::max(D, 3 * kT) * bt * sizeof(float);
  const size_t res = (size_t)kFC * kMaxOwnSegs * bt * sizeof(float);   // per-warp row sums
  const long long room = (long long)g_smem_optin - stat - (long long)(src + res);
  const int ring = (int)std::min<long long>(kMaxRing, room / kFStageBytes);
  if (ring < 2) return pl;
  pl.bt = bt;
  pl.groups = groups;
  pl.gsize = gsize;
  pl.grouped = grouped;
  pl.ring = ring;
  pl.smem = (size_t)ring * kFStageBytes + src + res;
  return pl;
}
}  // namespace

oda_status prepare_head_kernel() {
  // largest input tile: the tower phase with D = 8192 (Kc = 4096)
  oda_status st = check_cuda(cudaFuncSetAttribute(head_phase_kernel<8, 2>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  8 * 4096 * (int)sizeof(float)),
                             "cudaFuncSetAttribute(head)");
  if (st != ODA_OK) return st;
  st = check_cuda(cudaFuncSetAttribute(head_phase_kernel<4, 4>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       4 * 4096 * (int)sizeof(float)),
                  "cudaFuncSetAttribute(head)");
  if (st != ODA_OK) return st;
  int dev = 0;
  st = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (st == ODA_OK)
    st = check_cuda(cudaDeviceGetAttribute(&g_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev),
                    "cudaDeviceGetAttribute");
  if (st == ODA_OK)
    st = check_cuda(cudaDeviceGetAttribute(&g_coop, cudaDevAttrCooperativeLaunch, dev),
                    "cudaDeviceGetAttribute");
  if (st != ODA_OK) return st;
  for (int i = 0; i < 3; ++i) {
    const void* kern = reinterpret_cast<const void*>(fused_kernel(i));
    cudaFuncAttributes fa;
    st = check_cuda(cudaFuncGetAttributes(&fa, kern), "cudaFuncGetAttributes(head)");
    if (st != ODA_OK) return st;
    // 288 threads (9 warps, three on one SM sub-partition) allow at most 168 registers per thread;
    // a kernel built with more could never launch, every plan would fail and the phase kernels
    // would run in silence: refuse it here instead
    if (fa.maxThreadsPerBlock < kFThreads)
      return set_error(ODA_ERR_UNSUPPORTED, "fused recall head: %d registers per thread leave %d threads per block",
                       fa.numRegs, fa.maxThreadsPerBlock);
    g_fused_static[i] = (int)fa.sharedSizeBytes;
    st = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         g_smem_optin - g_fused_static[i]),
                    "cudaFuncSetAttribute(head)");
    if (st != ODA_OK) return st;
  }
  return ODA_OK;
}

// The path oda_recall_score takes for this context: the fused launch's tile width, sequence
// groups and ring depth, or zeros where the six phase kernels run.  Same plan and occupancy test
// as the launch below.
oda_status recall_head_plan(oda_ctx* ctx, int32_t* tile, int32_t* groups, int32_t* ring) {
  const FusedPlan pl = fused_plan(ctx->cfg.batch, ctx->cfg.head_in_dim, ctx->n_sms);
  int per_sm = 0;
  if (pl.bt) {
    const void* kern = reinterpret_cast<const void*>(fused_kernel(fused_index(pl.bt, pl.grouped)));
    const oda_status st = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFThreads, pl.smem),
                                     "cudaOccupancyMaxActiveBlocksPerMultiprocessor(head)");
    if (st != ODA_OK) return st;
  }
  const bool fused = pl.bt && per_sm >= 1;
  *tile = fused ? pl.bt : 0;
  *groups = fused ? pl.groups : 0;
  *ring = fused ? pl.ring : 0;
  return ODA_OK;
}

oda_status launch_recall_head(oda_ctx* ctx, const oda_head_weights* w, const float* h_prev,
                              const float* emb, const float* h_loc, const int32_t* sched,
                              float* score, int32_t* flag, int32_t* any_flag, cudaStream_t s) {
  if (!w || !h_prev || !emb || !h_loc || !score || !flag || !any_flag)
    return set_error(ODA_ERR_INVALID_ARG, "recall_score: null pointer argument");
  const void* ptrs[] = {w->fuse_w, w->fuse_b, w->out_norm, w->out_w, w->out_b};
  for (const void* q : ptrs)
    if (!q) return set_error(ODA_ERR_INVALID_ARG, "recall_score: null weight pointer");
  for (int i = 0; i < 3; ++i)
    if (!w->tower_norm[i] || !w->tower_w[i] || !w->tower_b[i])
      return set_error(ODA_ERR_INVALID_ARG, "recall_score: null tower weight pointer");
  for (int j = 0; j < 2; ++j)
    if (!w->ffn_norm[j] || !w->ffn_gate[j] || !w->ffn_up[j] || !w->ffn_down[j])
      return set_error(ODA_ERR_INVALID_ARG, "recall_score: null FFN weight pointer");
  const void* mats[] = {w->tower_w[0], w->tower_w[1], w->tower_w[2], w->fuse_w, w->ffn_gate[0],
                        w->ffn_gate[1], w->ffn_up[0], w->ffn_up[1], w->ffn_down[0], w->ffn_down[1],
                        h_prev, emb, h_loc};
  for (const void* q : mats)
    if (reinterpret_cast<uintptr_t>(q) & 15)
      return set_error(ODA_ERR_INVALID_ARG, "recall_score: matrices and inputs must be 16-byte aligned");
  const int B = ctx->cfg.batch, D = ctx->cfg.head_in_dim;
  // One cooperative launch for the whole batch: groups of up to 8 sequences, each on its own
  // share of the SMs, all groups in step (one grid barrier per phase).  CTA i of every group
  // streams the same weight segments at about the same time, so HBM serves each segment once and
  // L2 the other groups.
  const FusedPlan pl = fused_plan(B, D, ctx->n_sms);
  int per_sm = 0;
  if (pl.bt) {
    const void* kern = reinterpret_cast<const void*>(fused_kernel(fused_index(pl.bt, pl.grouped)));
    oda_status st = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFThreads, pl.smem),
                               "cudaOccupancyMaxActiveBlocksPerMultiprocessor(head)");
    if (st != ODA_OK) return st;
  }
  if (pl.bt && per_sm >= 1) {
    // one CTA per SM, all resident at once (cooperative launch): the grid barrier needs that
    FusedParams f;
    f.w = *w;
    f.x[0] = h_prev;
    f.x[1] = emb;
    f.x[2] = h_loc;
    f.sched = sched;
    f.score = score;
    f.flag = flag;
    f.any_flag = any_flag;
    f.u = ctx->head_u;
    f.f = ctx->head_f;
    f.act = ctx->head_act;
    f.cnt = ctx->head_cnt;
    f.err = ctx->err;
    f.B = B;
    f.D = D;
    f.ring = pl.ring;
    f.groups = pl.groups;
    f.gsize = pl.gsize;
    f.theta = ctx->cfg.theta;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(ctx->n_sms);
    lc.blockDim = dim3(kFThreads);
    lc.dynamicSmemBytes = pl.smem;
    lc.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return check_cuda(cudaLaunchKernelEx(&lc, fused_kernel(fused_index(pl.bt, pl.grouped)), f),
                      "recall head launch");
  }
  HeadParams p;
  p.w = *w;
  p.x[0] = h_prev;
  p.x[1] = emb;
  p.x[2] = h_loc;
  p.sched = sched;
  p.score = score;
  p.flag = flag;
  p.any_flag = any_flag;
  p.part = ctx->head_part;
  p.ss = ctx->head_ss;
  p.cnt = ctx->head_cnt;
  p.u = ctx->head_u;
  p.f = ctx->head_f;
  p.act = ctx->head_act;
  p.B = ctx->cfg.batch;
  p.D = ctx->cfg.head_in_dim;
  p.theta = ctx->cfg.theta;
  const int seq[6][2] = {{kTower, 0}, {kFuse, 0}, {kUp, 0}, {kDown, 0}, {kUp, 1}, {kDown, 1}};
  for (int i = 0; i < 6; ++i) {
    p.phase = seq[i][0];
    p.block = seq[i][1];
    const PhaseShape sh = phase_shape(p.phase, p.D);
    p.Kc = sh.Kc;
    p.nchunks = sh.nchunks;
    p.rows_total = sh.rows_total;
    p.row_blocks = sh.row_blocks;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(sh.row_blocks * sh.nchunks);
    lc.blockDim = dim3(kHT);
    const int bt = p.B <= 4 ? 4 : kBTMax;
    lc.dynamicSmemBytes = bt * sh.Kc * sizeof(float);
    lc.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    oda_status st = check_cuda(bt == 4 ? cudaLaunchKernelEx(&lc, head_phase_kernel<4, 4>, p)
                                       : cudaLaunchKernelEx(&lc, head_phase_kernel<8, 2>, p),
                               "recall head launch");
    if (st != ODA_OK) return st;
  }
  return ODA_OK;
}

}  // namespace oda
