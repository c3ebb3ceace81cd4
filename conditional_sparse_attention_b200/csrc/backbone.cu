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


constexpr int kXPad = 8;            // bf16 padding of an input row (rows 4 banks apart)
// Packed weight layout (oda_bb_pack_weight): blocks of 16 rows x 512 columns (16 KiB), tile-major
// then column-block; inside a block row r holds its 64 16-byte chunks with chunk j at slot
// j ^ (r & 7), so the 8 rows an ldmatrix reads at one column fall in 8 distinct bank groups.
constexpr int kBlkCols = 512;
constexpr int kBlkElems = kTile * kBlkCols;          // 8192
constexpr int kBlkBytes = kBlkElems * 2;             // 16 KiB
constexpr int kPiece = 8192;                         // bytes per bulk copy of a stage
constexpr int kGThreads = (kBW + 1) * 32;   // 8 consumer warps + 1 producer warp
constexpr int kMaxRing = 6;
constexpr uint64_t kGWaitNs = 2000000000ull;

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kBW * 32) : "memory");
}

// One projection phase: out = W in (N x K, bf16 weights, the batch's B input rows), with its input
// staging and its epilogue.  A launch runs one phase, or - the fused post-attention launch - the
// four phases between two attention layers, separated by grid barriers.
struct Phase {
  const uint16_t* W;      // [N][K] bf16 (the gate projection for kEpiGateUp)
  const uint16_t* W2;     // kEpiGateUp: the up projection [N][K]
  const float* gamma;     // kInNorm: [K]
  const float* xf;        // kInNorm / kInF32: [B][K] fp32
  const uint16_t* xb;     // kInBf16: [B][K] bf16
  float* out_f;           // kEpiResid: the residual [B][N] (+= W in); kEpiLogits: [B][N]
  uint16_t* out_b;        // kEpiGateUp: act [B][N]; kEpiQKV: q [B][Hq*128]
  uint16_t* kn;           // kEpiQKV: [B][Hkv*128]
  uint16_t* vn;
  int K, N, kst, epi, in;   // kst: K values per ring stage (a K chunk of one tile)
};

constexpr int kMaxPhases = 4;

struct ProjParams {
  Phase ph[kMaxPhases];
  int n_ph;
  int32_t* cnt;           // n_ph > 1: [0] grid-barrier arrivals, [1] finished CTAs (0 at exit)
  int32_t* err;
  int B, Hq, Hkv;
  int R, stage_bytes, ldx_cap;   // ring stages, bytes per stage, bf16 pitch of the widest input
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Loads the B input rows of phase P (K values each) into xs as bf16 (row pitch ldx):
// kInNorm bf16(x * rsqrt(mean(x^2) + eps) * gamma), kInF32 bf16(x), kInBf16 a copy (gamma
// already in shared memory: s_gamma, loaded by load_gamma before a barrier).  A thread
// issues every load of a round (up to 4 vectors) before using any: the inputs are a few KB, so
// staging costs dependent round trips to L2, not bandwidth.  Loads bypass L1 (in the fused
// launch other CTAs wrote the inputs).  The sums of squares are added in a fixed order: per
// warp (32 consecutive float4 of one row, since K % 512 == 0) by shuffles, those warp sums in
// round order, then the 8 warps' partials in warp order.  Called by the 256 consumer threads;
// ends with their barrier.
__device__ __forceinline__ void stage_input(const Phase& P, uint16_t* xs, int ldx, int B,
                                            float (*s_part)[kMaxB], float* s_inv, const float* s_gamma,
                                            int tid) {
  constexpr int kT = kBW * 32, kU = 4;
  const int K = P.K;
  if (P.in == kInBf16) {
    const int per_row = K / 8, n = B * per_row;
    const uint4* src = reinterpret_cast<const uint4*>(P.xb);
    for (int base = 0; base < n; base += kU * kT) {
      uint4 v[kU];
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int u = base + j * kT + tid;
        if (u < n) v[j] = __ldcg(src + u);
      }
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int u = base + j * kT + tid;
        if (u < n) {
          const int b = u / per_row, c = u - b * per_row;
          *reinterpret_cast<uint4*>(xs + (size_t)b * ldx + 8 * c) = v[j];
        }
      }
    }
    consumers_sync();
    return;
  }
  const int per_row = K / 4, n = B * per_row;
  const float4* src = reinterpret_cast<const float4*>(P.xf);
  const float4* g4 = reinterpret_cast<const float4*>(s_gamma);
  const bool norm = P.in == kInNorm;
  const int warp = tid >> 5, lane = tid & 31;
  if (n <= kU * kT) {
    // one round trip: the values stay in registers between the sums of squares and the store
    float4 v[kU];
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int u = j * kT + tid;
      if (u < n) v[j] = __ldcg(src + u);
    }
    if (norm) {
      if (lane < kMaxB) s_part[warp][lane] = 0.f;
      __syncwarp();
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int u0 = j * kT + warp * 32;
        if (u0 < n) {
          float ss = fmaf(v[j].x, v[j].x, 0.f);
          ss = fmaf(v[j].y, v[j].y, ss);
          ss = fmaf(v[j].z, v[j].z, ss);
          ss = fmaf(v[j].w, v[j].w, ss);
          ss = warp_sum(ss);
          if (lane == 0) s_part[warp][u0 / per_row] += ss;
        }
      }
      consumers_sync();
    }
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int u = j * kT + tid;
      if (u < n) {
        const int b = u / per_row, c = u - b * per_row;
        float4 y = v[j];
        if (norm) {
          float ss = 0.f;
#pragma unroll
          for (int w = 0; w < kBW; ++w) ss += s_part[w][b];
          const float r = rsqrtf(ss / (float)K + kEps);
          const float4 gg = g4[c];
          y.x = y.x * r * gg.x;
          y.y = y.y * r * gg.y;
          y.z = y.z * r * gg.z;
          y.w = y.w * r * gg.w;
        }
        uint2 w;
        w.x = (uint32_t)f32_to_bf16_bits(y.x) | ((uint32_t)f32_to_bf16_bits(y.y) << 16);
        w.y = (uint32_t)f32_to_bf16_bits(y.z) | ((uint32_t)f32_to_bf16_bits(y.w) << 16);
        *reinterpret_cast<uint2*>(xs + (size_t)b * ldx + 4 * c) = w;
      }
    }
    consumers_sync();
    return;
  }
  if (norm) {
    if (lane < kMaxB) s_part[warp][lane] = 0.f;
    __syncwarp();
    for (int base = 0; base < n; base += kU * kT) {
      float4 v[kU];
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int u = base + j * kT + tid;
        if (u < n) v[j] = __ldcg(src + u);
      }
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int u0 = base + j * kT + warp * 32;   // the warp's first vector: all in or all out
        if (u0 < n) {
          float ss = fmaf(v[j].x, v[j].x, 0.f);
          ss = fmaf(v[j].y, v[j].y, ss);
          ss = fmaf(v[j].z, v[j].z, ss);
          ss = fmaf(v[j].w, v[j].w, ss);
          ss = warp_sum(ss);
          if (lane == 0) s_part[warp][u0 / per_row] += ss;
        }
      }
    }
    consumers_sync();
    if (tid < B) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < kBW; ++w) ss += s_part[w][tid];
      s_inv[tid] = rsqrtf(ss / (float)K + kEps);
    }
    consumers_sync();
  }
  for (int base = 0; base < n; base += kU * kT) {
    float4 v[kU];
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int u = base + j * kT + tid;
      if (u < n) v[j] = __ldcg(src + u);
    }
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int u = base + j * kT + tid;
      if (u < n) {
        const int b = u / per_row, c = u - b * per_row;
        float4 y = v[j];
        if (norm) {
          const float r = s_inv[b];
          const float4 gg = g4[c];
          y.x = y.x * r * gg.x;
          y.y = y.y * r * gg.y;
          y.z = y.z * r * gg.z;
          y.w = y.w * r * gg.w;
        }
        uint2 w;
        w.x = (uint32_t)f32_to_bf16_bits(y.x) | ((uint32_t)f32_to_bf16_bits(y.y) << 16);
        w.y = (uint32_t)f32_to_bf16_bits(y.z) | ((uint32_t)f32_to_bf16_bits(y.w) << 16);
        *reinterpret_cast<uint2*>(xs + (size_t)b * ldx + 4 * c) = w;
      }
    }
  }
  consumers_sync();
}

// One ring stage of a tile (16 weight rows, or the 16 gate rows then the 16 up rows, in packed
// blocks; this warp's kw columns from c0) against the inputs: A fragments of the weight rows and
// B fragments of the input rows by ldmatrix, mma.sync bf16 -> fp32.  up_blk: the stage's first
// block of up rows.  xrow: this lane's input row (batch rr = lane & 7) in xs, or - rows b >= B -
// a 16-byte zero block read for every column.
__device__ __forceinline__ uint32_t packed_addr(uint32_t sb, int blk0, int row, int col) {
  return sb + (uint32_t)(((blk0 + (col >> 9)) * kBlkBytes) + (row << 10) + ((((col & 511) >> 3) ^ (row & 7)) << 4));
}

// gamma of a normalising phase into shared memory (it does not depend on earlier kernels or
// phases, so it is loaded before the wait for them).  The reader is behind a consumer barrier.
__device__ __forceinline__ void load_gamma(const Phase& P, float* s_gamma, int tid) {
  if (P.in != kInNorm) return;
  const float4* g = reinterpret_cast<const float4*>(P.gamma);
  for (int i = tid; i < P.K / 4; i += kBW * 32) reinterpret_cast<float4*>(s_gamma)[i] = __ldg(g + i);
}

// NIT groups of 32 columns per warp and stage (kst / 8 / 32).  All of a stage's fragments are
// loaded before the first product, and the two 16-column halves of a group accumulate in two
// independent chains (acc[0], acc[1]; added at the end of the tile), so a warp's stage costs
// about one ldmatrix latency plus NIT dependent products instead of a serial chain of both.
template <int NIT, bool GU>
__device__ __forceinline__ void consume_stage(float (&acc)[2][4], float (&accu)[2][4], uint32_t sb, int up_blk,
                                              uint32_t xrow, bool xvalid, int col_x, int c0, int lane) {
  const int mi = lane >> 3, rr = lane & 7;
  const int arow = ((mi & 1) << 3) + rr, acol = (mi >> 1) << 3;
  const int bcol = mi << 3;
  uint32_t xb[NIT][4], a[NIT][2][4], au[GU ? NIT : 1][2][4];
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    ldsm_x4(xb[it], xvalid ? xrow + (col_x + 32 * it + bcol) * 2 : xrow);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = c0 + 32 * it + 16 * h + acol;
      ldsm_x4(a[it][h], packed_addr(sb, 0, arow, col));
      if (GU) ldsm_x4(au[GU ? it : 0][h], packed_addr(sb, up_blk, arow, col));
    }
  }
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mma_bf16_16816(acc[h], a[it][h], xb[it][2 * h], xb[it][2 * h + 1]);
      if (GU) mma_bf16_16816(accu[h], au[GU ? it : 0][h], xb[it][2 * h], xb[it][2 * h + 1]);
    }
  }
}

// The warps' column shares of a finished tile, added in warp order, and the phase's epilogue.
// Lane (g, c) of a warp holds rows g, g + 8 and sequences 2c, 2c + 1.  red is double-buffered
// by tile parity (buf), so one barrier per tile suffices: buffer buf is written again two tiles
// later, after the next tile's barrier, which every reader of this tile has passed.  r_old: the
// residual element of this thread's (row, sequence), loaded before the tile's stages.
// red: per buffer [warp][gate | up][16 rows][B]
__host__ __device__ constexpr int red_floats(int B) { return kBW * 2 * kTile * B; }

__device__ __forceinline__ void tile_epilogue(const Phase& P, const ProjParams& p, float* red, int buf,
                                              const float (&acc)[2][4], const float (&accu)[2][4], int t,
                                              int warp, int lane, int tid, float r_old) {
  const int g = lane >> 2, c = lane & 3, B = p.B;
  const bool gu = P.epi == kEpiGateUp;
  float* rb = red + (size_t)buf * red_floats(B);
  float* rw = rb + (size_t)warp * 2 * kTile * B;
  if (2 * c < B) {
    rw[g * B + 2 * c] = acc[0][0] + acc[1][0];
    rw[(g + 8) * B + 2 * c] = acc[0][2] + acc[1][2];
    if (gu) {
      rw[kTile * B + g * B + 2 * c] = accu[0][0] + accu[1][0];
      rw[kTile * B + (g + 8) * B + 2 * c] = accu[0][2] + accu[1][2];
    }
  }
  if (2 * c + 1 < B) {
    rw[g * B + 2 * c + 1] = acc[0][1] + acc[1][1];
    rw[(g + 8) * B + 2 * c + 1] = acc[0][3] + acc[1][3];
    if (gu) {
      rw[kTile * B + g * B + 2 * c + 1] = accu[0][1] + accu[1][1];
      rw[kTile * B + (g + 8) * B + 2 * c + 1] = accu[0][3] + accu[1][3];
    }
  }
  consumers_sync();
  if (tid < kTile * B) {
    const int row = tid / B, b = tid - row * B;
    {
      float y = 0.f, yu = 0.f;
#pragma unroll
      for (int ww = 0; ww < kBW; ++ww) {
        y += rb[(size_t)ww * 2 * kTile * B + tid];
        if (gu) yu += rb[(size_t)ww * 2 * kTile * B + kTile * B + tid];
      }
      const int n = t * kTile + row;
      if (P.epi == kEpiQKV) {
        const int nq = p.Hq * 128, nk = p.Hkv * 128;
        const uint16_t v = f32_to_bf16_bits(y);
        if (n < nq) P.out_b[(size_t)b * nq + n] = v;
        else if (n < nq + nk) P.kn[(size_t)b * nk + (n - nq)] = v;
        else P.vn[(size_t)b * nk + (n - nq - nk)] = v;
      } else if (P.epi == kEpiResid) {
        P.out_f[(size_t)b * P.N + n] = r_old + y;
      } else if (gu) {
        const float sl = y / (1.0f + expf(-y));
        P.out_b[(size_t)b * P.N + n] = f32_to_bf16_bits(sl * yu);
      } else {
        P.out_f[(size_t)b * P.N + n] = y;
      }
    }
  }
}

// Persistent projection kernel: one CTA per SM takes tiles t = blockIdx.x, + gridDim.x, ... of
// each phase.  A producer warp streams every (phase, tile, K chunk) of its CTA, in order, through
// a ring of shared-memory stages with one bulk copy per row segment (completion counted on the
// stage's mbarrier).  It only reads weights, which no phase writes, so it runs ahead of the
// consumers - into the next phase while they wait at a grid barrier, and before the previous
// kernel has finished.  The 8 consumer warps each take 1/8 of every chunk's columns; at the end
// of a tile their partial sums are added in warp order and the epilogue writes the outputs, so
// every output element has one writer and a fixed summation order.  With more than one phase
// the launch is cooperative and a bounded grid barrier separates the phases.
__global__ void __launch_bounds__(kGThreads, 1) bb_proj_kernel(const ProjParams p) {
  extern __shared__ __align__(128) uint8_t bsm[];
  const int R = p.R;
  uint8_t* stages = bsm;
  uint16_t* xs = reinterpret_cast<uint16_t*>(bsm + (size_t)R * p.stage_bytes);        // [B][ldx]
  float* red = reinterpret_cast<float*>(bsm + (size_t)R * p.stage_bytes + (size_t)p.B * p.ldx_cap * 2);
  float* s_gamma = red + 2 * red_floats(p.B);                                           // [K of a norm]
  __shared__ __align__(8) uint64_t full[kMaxRing];
  __shared__ __align__(8) uint64_t empty[kMaxRing];
  __shared__ __align__(16) uint4 s_zero;
  __shared__ float s_part[kBW][kMaxB];
  __shared__ float s_inv[kMaxB];
  __shared__ Phase s_ph[kMaxPhases];   // the phases, indexed by a runtime phase number
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
#pragma unroll
  for (int i = 0; i < kMaxPhases; ++i)
    if (tid == 32 * i + 1) s_ph[i] = p.ph[i];
  if (tid == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kBW);
    }
    fence_mbar_init();
    s_zero = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  if (warp == kBW) {
    // ---- producer
    int k = 0;
    for (int ph = 0; ph < p.n_ph; ++ph) {
      const Phase& P = s_ph[ph];
      const int rows = P.epi == kEpiGateUp ? 2 * kTile : kTile;
      const int nck = P.K / P.kst, nb = P.K / kBlkCols;
      const int w_bytes = kTile * P.kst * 2;        // bytes of W (and of W2) per stage
      const int np_w = w_bytes / kPiece, np = rows == kTile ? np_w : 2 * np_w;
      for (int t = blockIdx.x; t < P.N / kTile; t += G) {
        for (int ch = 0; ch < nck; ++ch, ++k) {
          const int s = k % R;
          if (k >= R && !mbar_wait_bounded(&empty[s], (uint32_t)(k / R - 1) & 1u, kGWaitNs)) {
            if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
            return;
          }
          if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(rows * P.kst * 2));
          __syncwarp();
          if (lane < np) {
            // the chunk's blocks of a tile are contiguous: one range per matrix, in 8 KiB copies
            const bool up = lane >= np_w;
            const int i = up ? lane - np_w : lane;
            const size_t blk = (size_t)t * nb + (size_t)ch * (P.kst / kBlkCols);
            const uint16_t* src = (up ? P.W2 : P.W) + blk * kBlkElems + (size_t)i * (kPiece / 2);
            bulk_load(stages + (size_t)s * p.stage_bytes + (up ? w_bytes : 0) + (size_t)i * kPiece, src,
                      (uint32_t)kPiece, &full[s]);
          }
        }
      }
    }
    return;
  }

  // ---- consumers
  load_gamma(s_ph[0], s_gamma, tid);
  grid_dependency_wait();
  grid_dependents_launch();
  const int rr = lane & 7;
  const bool xvalid = rr < p.B;
  const uint32_t zero_addr = smem_u32(&s_zero);
  int k = 0, n_tiles_done = 0;
  for (int ph = 0; ph < p.n_ph; ++ph) {
    const Phase& P = s_ph[ph];
    const int K = P.K, kst = P.kst, nck = K / kst, kw = kst / kBW, up_blk = kst / kBlkCols;
    const int ldx = K + kXPad;
    if (ph > 0) {
      // every CTA's outputs of the previous phase are complete and visible: the CTA's barrier
      // orders its threads' stores before thread 0's release (cumulative), and thread 0's acquire
      // before the other threads' loads
      consumers_sync();
      if (tid == 0 && !grid_barrier_bounded(p.cnt, ph * G, kGWaitNs)) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
      consumers_sync();
    }
    const bool has_tiles = (int)blockIdx.x < P.N / kTile;
    if (has_tiles) stage_input(P, xs, ldx, p.B, s_part, s_inv, s_gamma, tid);
    // the next phase's gamma, read behind its barrier, arrives during this phase's tiles
    if (ph + 1 < p.n_ph) load_gamma(s_ph[ph + 1], s_gamma, tid);
    if (!has_tiles) continue;
    const uint32_t xrow = xvalid ? smem_u32(xs) + (uint32_t)(rr * ldx) * 2u : zero_addr;
    const int erow = tid / p.B, eb = tid - erow * p.B;   // this thread's epilogue element
    for (int t = blockIdx.x; t < P.N / kTile; t += G, ++n_tiles_done) {
      float r_old = 0.f;
      if (P.epi == kEpiResid && tid < kTile * p.B)
        r_old = __ldcg(P.out_f + (size_t)eb * P.N + t * kTile + erow);
      float acc[2][4] = {}, accu[2][4] = {};
      for (int ch = 0; ch < nck; ++ch, ++k) {
        const int s = k % R;
        if (!mbar_wait_bounded(&full[s], (uint32_t)(k / R) & 1u, kGWaitNs)) {
          if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
        }
        const uint32_t sb = smem_u32(stages + (size_t)s * p.stage_bytes);
        const int c0 = warp * kw;
        if (P.epi == kEpiGateUp)   // kst = 512: 64 columns per warp
          consume_stage<2, true>(acc, accu, sb, up_blk, xrow, xvalid, ch * kst + c0, c0, lane);
        else if (kw == 128)
          consume_stage<4, false>(acc, accu, sb, up_blk, xrow, xvalid, ch * kst + c0, c0, lane);
        else
          consume_stage<2, false>(acc, accu, sb, up_blk, xrow, xvalid, ch * kst + c0, c0, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      tile_epilogue(P, p, red, n_tiles_done & 1, acc, accu, t, warp, lane, tid, r_old);
    }
  }
  if (p.n_ph > 1) {
    // the last CTA to finish returns the barrier counters to zero (every CTA has passed every
    // barrier before it counts itself finished)
    consumers_sync();
    if (tid == 0 && atom_add_acq_rel_gpu(p.cnt + 1, 1) == G - 1) {
      p.cnt[0] = 0;
      p.cnt[1] = 0;
    }
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
  // row t of the packed table: block (t / 16, kk / 512), row t % 16, swizzled 16-byte chunk
  const size_t row0 = (size_t)(t >> 4) * (D / kBlkCols) * kBlkElems + (size_t)(t & 15) * kBlkCols;
  for (int kk = threadIdx.x; kk < D; kk += blockDim.x) {
    const size_t e = row0 + (size_t)(kk >> 9) * kBlkElems + ((((kk & 511) >> 3) ^ (t & 7)) << 3) + (kk & 7);
    emb[(size_t)b * D + kk] = __uint_as_float((uint32_t)E[e] << 16);
  }
}

// dst = src [rows][cols] bf16 (row-major) in the packed layout; one thread per 16-byte chunk.
__global__ void bb_pack_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int rows, int cols) {
  const int cpr = cols / 8;   // chunks per row
  const size_t n = (size_t)rows * cpr;
  for (size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x; q < n; q += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(q / cpr), j = (int)(q - (size_t)r * cpr);
    const size_t blk = (size_t)(r >> 4) * (cols / kBlkCols) + (j >> 6);
    dst[blk * (kBlkElems / 8) + (size_t)(r & 15) * (kBlkCols / 8) + ((j & 63) ^ (r & 7))] = src[q];
  }
}

int g_bb_smem_optin = 0;

// Launches phases ph[0 .. n - 1] of one projection launch: a single phase as an ordinary
// persistent launch (overlapping the previous kernel when the context allows), several as one
// cooperative launch of one CTA per SM.  The ring takes the shared memory left after the input
// rows (B of them, as wide as the widest input) and the reduction area.
oda_status launch_proj(oda_ctx* ctx, const Phase* ph, int n, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  ProjParams p = {};
  p.n_ph = n;
  p.err = ctx->err;
  p.B = cf.batch;
  p.Hq = cf.n_q_heads;
  p.Hkv = cf.n_kv_heads;
  int max_k = 0, n_tiles = 0, norm_k = 0;
  for (int i = 0; i < n; ++i) {
    p.ph[i] = ph[i];
    Phase& P = p.ph[i];
    // a stage of about 32 KiB: 1024 columns of 16 rows, or 512 of the gate and up rows together
    P.kst = (P.epi != kEpiGateUp && P.K % 1024 == 0) ? 1024 : 512;
    const int rows = P.epi == kEpiGateUp ? 2 * kTile : kTile;
    p.stage_bytes = std::max(p.stage_bytes, rows * P.kst * 2);
    max_k = std::max(max_k, P.K);
    if (P.in == kInNorm) norm_k = std::max(norm_k, P.K);
    n_tiles = std::max(n_tiles, P.N / kTile);
  }
  p.ldx_cap = max_k + kXPad;
  const size_t fixed = (size_t)cf.batch * p.ldx_cap * 2 + 2 * (size_t)red_floats(cf.batch) * 4 + (size_t)norm_k * 4;
  const long long room = (long long)g_bb_smem_optin - 1024 - (long long)fixed;
  p.R = (int)std::min<long long>(kMaxRing, room / p.stage_bytes);
  if (p.R < 2) return set_error(ODA_ERR_UNSUPPORTED, "backbone: input width %d needs more shared memory", max_k);
  const size_t smem = (size_t)p.R * p.stage_bytes + fixed;
  static int attr_set = 0;   // the kernel's dynamic shared-memory limit, raised once to the opt-in
  if (!attr_set) {
    oda_status st = check_cuda(cudaFuncSetAttribute(bb_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    g_bb_smem_optin - 1024),
                               "cudaFuncSetAttribute(backbone)");
    if (st != ODA_OK) return st;
    attr_set = 1;
  }
  cudaLaunchConfig_t lc = {};
  lc.blockDim = dim3(kGThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[2];
  if (n == 1) {
    lc.gridDim = dim3(std::min(n_tiles, ctx->n_sms));
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.numAttrs = cf.overlap_layers ? 1 : 0;
  } else {
    int coop = 0, dev = 0, per_sm = 0;
    oda_status st = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
    if (st == ODA_OK)
      st = check_cuda(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev), "cudaDeviceGetAttribute");
    if (st == ODA_OK)
      st = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bb_proj_kernel, kGThreads, smem),
                      "cudaOccupancyMaxActiveBlocksPerMultiprocessor(backbone)");
    if (st != ODA_OK) return st;
    if (!coop) return set_error(ODA_ERR_UNSUPPORTED, "backbone: the device has no cooperative launch");
    if (per_sm < 1) return set_error(ODA_ERR_UNSUPPORTED, "backbone: the fused launch does not fit on an SM");
    p.cnt = ctx->bb_cnt + ctx->bb_cnt_n - 2;   // the last two counters: barrier, finished CTAs
    lc.gridDim = dim3(ctx->n_sms);
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.numAttrs = 1;
    if (cf.overlap_layers) {
      // the producers stream weights (which no earlier kernel writes) while the previous
      // kernel finishes; the consumers wait for it before reading any input.  CTAs that find
      // no free SM yet are placed as the previous kernel's CTAs leave (they wait on nothing of
      // this launch), so all of them become resident before any grid barrier can complete.
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      lc.numAttrs = 2;
    }
  }
  lc.attrs = attr;
  oda_status st = check_cuda(cudaLaunchKernelEx(&lc, bb_proj_kernel, p), "backbone projection launch");
  ctx->prev_attention = (st == ODA_OK);
  return st;
}

Phase phase_qkv(const oda_bb_layer* w, const float* x, void* q, void* k_new, void* v_new, int D, int N) {
  Phase P = {};
  P.W = static_cast<const uint16_t*>(w->w_qkv);
  P.gamma = w->attn_norm;
  P.xf = x;
  P.out_b = static_cast<uint16_t*>(q);
  P.kn = static_cast<uint16_t*>(k_new);
  P.vn = static_cast<uint16_t*>(v_new);
  P.K = D;
  P.N = N;
  P.epi = kEpiQKV;
  P.in = kInNorm;
  return P;
}

Phase phase_o(const oda_bb_layer* w, const float* o, float* x, int D) {
  Phase P = {};
  P.W = static_cast<const uint16_t*>(w->w_o);
  P.xf = o;
  P.out_f = x;
  P.K = D;
  P.N = D;
  P.epi = kEpiResid;
  P.in = kInF32;
  return P;
}

Phase phase_gate_up(const oda_bb_layer* w, const float* x, void* act, int D, int F) {
  Phase P = {};
  P.W = static_cast<const uint16_t*>(w->w_gate);
  P.W2 = static_cast<const uint16_t*>(w->w_up);
  P.gamma = w->mlp_norm;
  P.xf = x;
  P.out_b = static_cast<uint16_t*>(act);
  P.K = D;
  P.N = F;
  P.epi = kEpiGateUp;
  P.in = kInNorm;
  return P;
}

Phase phase_down(const oda_bb_layer* w, const void* act, float* x, int D, int F) {
  Phase P = {};
  P.W = static_cast<const uint16_t*>(w->w_down);
  P.xb = static_cast<const uint16_t*>(act);
  P.out_f = x;
  P.K = F;
  P.N = D;
  P.epi = kEpiResid;
  P.in = kInBf16;
  return P;
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
  if (misaligned(w->w_qkv) || misaligned(x) || misaligned(w->attn_norm))
    return set_error(ODA_ERR_INVALID_ARG, "bb_qkv: weights and x must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, N, "bb_qkv");
  if (st != ODA_OK) return st;
  const Phase P = phase_qkv(w, x, q, k_new, v_new, D, N);
  return launch_proj(ctx, &P, 1, s);
}

oda_status launch_bb_attn_out(oda_ctx* ctx, const oda_bb_layer* w, const float* o, float* x, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128;
  if (!w || !w->w_o || !o || !x) return set_error(ODA_ERR_INVALID_ARG, "bb_attn_out: null pointer argument");
  if (misaligned(w->w_o) || misaligned(o) || misaligned(x))
    return set_error(ODA_ERR_INVALID_ARG, "bb_attn_out: weights, o and x must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, D, "bb_attn_out");
  if (st != ODA_OK) return st;
  const Phase P = phase_o(w, o, x, D);
  return launch_proj(ctx, &P, 1, s);
}

oda_status launch_bb_mlp(oda_ctx* ctx, const oda_bb_layer* w, float* x, void* act, cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128, F = w ? w->ffn : 0;
  if (!w || !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down || !x || !act)
    return set_error(ODA_ERR_INVALID_ARG, "bb_mlp: null pointer argument");
  if (misaligned(w->w_gate) || misaligned(w->w_up) || misaligned(w->w_down) || misaligned(x) ||
      misaligned(act) || misaligned(w->mlp_norm))
    return set_error(ODA_ERR_INVALID_ARG, "bb_mlp: weights, x and act must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, F, "bb_mlp(gate/up)");
  if (st == ODA_OK) st = check_shapes(ctx, F, D, "bb_mlp(down)");
  if (st != ODA_OK) return st;
  const Phase gu = phase_gate_up(w, x, act, D, F);
  st = launch_proj(ctx, &gu, 1, s);
  if (st != ODA_OK) return st;
  const Phase dn = phase_down(w, act, x, D, F);
  return launch_proj(ctx, &dn, 1, s);
}

oda_status launch_bb_post(oda_ctx* ctx, const oda_bb_layer* w, const oda_bb_layer* next,
                          const float* o, float* x, void* act, void* q, void* k_new, void* v_new,
                          cudaStream_t s) {
  const oda_config& cf = ctx->cfg;
  const int D = cf.n_q_heads * 128, F = w ? w->ffn : 0;
  const int Nqkv = (cf.n_q_heads + 2 * cf.n_kv_heads) * 128;
  if (!w || !w->w_o || !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down || !o || !x || !act)
    return set_error(ODA_ERR_INVALID_ARG, "bb_post: null pointer argument");
  if (next && (!next->attn_norm || !next->w_qkv || !q || !k_new || !v_new))
    return set_error(ODA_ERR_INVALID_ARG, "bb_post: null pointer argument for the next layer");
  const void* al[] = {w->w_o, w->w_gate, w->w_up, w->w_down, w->mlp_norm, o, x, act,
                      next ? next->w_qkv : nullptr, next ? next->attn_norm : nullptr};
  for (const void* a : al)
    if (misaligned(a)) return set_error(ODA_ERR_INVALID_ARG, "bb_post: weights and buffers must be 16-byte aligned");
  oda_status st = check_shapes(ctx, D, D, "bb_post(o)");
  if (st == ODA_OK) st = check_shapes(ctx, D, F, "bb_post(gate/up)");
  if (st == ODA_OK) st = check_shapes(ctx, F, D, "bb_post(down)");
  if (st == ODA_OK && next) st = check_shapes(ctx, D, Nqkv, "bb_post(qkv)");
  if (st != ODA_OK) return st;
  Phase ph[kMaxPhases] = {phase_o(w, o, x, D), phase_gate_up(w, x, act, D, F), phase_down(w, act, x, D, F)};
  int n = 3;
  if (next) ph[n++] = phase_qkv(next, x, q, k_new, v_new, D, Nqkv);
  return launch_proj(ctx, ph, n, s);
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
  Phase P = {};
  P.W = static_cast<const uint16_t*>(embed);
  P.xf = h;
  P.out_f = logits;
  P.K = D;
  P.N = vocab;
  P.epi = kEpiLogits;
  P.in = kInF32;
  st = launch_proj(ctx, &P, 1, s);
  if (st != ODA_OK) return st;
  const int nsl = std::max(1, std::min(64, vocab / 2048));
  float* part_v = ctx->bb_part;
  int32_t* part_i = reinterpret_cast<int32_t*>(ctx->bb_part + (size_t)cf.batch * nsl);
  return launch_small(ctx, bb_argmax_embed_kernel, dim3(nsl, cf.batch), dim3(256), s, "bb_argmax launch",
                      (const float*)logits, (int)vocab, (const int32_t*)nullptr, token,
                      static_cast<const uint16_t*>(embed), next_emb, D, part_v, part_i, ctx->bb_cnt);
}

oda_status launch_bb_pack_weight(oda_ctx* ctx, const void* src, int32_t rows, int32_t cols, void* dst,
                                 cudaStream_t s) {
  if (!src || !dst) return set_error(ODA_ERR_INVALID_ARG, "bb_pack_weight: null pointer argument");
  if (src == dst) return set_error(ODA_ERR_INVALID_ARG, "bb_pack_weight: src and dst must not overlap");
  if (misaligned(src) || misaligned(dst))
    return set_error(ODA_ERR_INVALID_ARG, "bb_pack_weight: src and dst must be 16-byte aligned");
  if (rows < kTile || rows % kTile != 0 || cols < kBlkCols || cols % kBlkCols != 0)
    return set_error(ODA_ERR_INVALID_ARG, "bb_pack_weight: need rows a multiple of 16 and cols of 512 (%d x %d)",
                     rows, cols);
  const size_t n = (size_t)rows * (cols / 8);
  const int grid = (int)std::min<size_t>((n + 255) / 256, (size_t)ctx->n_sms * 8);
  bb_pack_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, cols);
  ctx->prev_attention = false;
  return check_cuda(cudaGetLastError(), "bb_pack_weight launch");
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
