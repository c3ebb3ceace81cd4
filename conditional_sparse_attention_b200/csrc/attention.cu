// Split-KV flash-decode over a paged bf16 KV cache for the two ODA index sets.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.1, eq. o_t and
// eq. S^F / S^L: one decode query per sequence attends, per layer, over either the local set
// S^L_t = {1..min(s,t)} U {max(1,t-w+1)..t} or the full set S^F_t = {1..t} of one retained
// cache; the current token's K,V (position t) come from the branch's staging, not the cache.
//
// Shared per-page arithmetic (sm_100a):
//   * every warp streams its pages through a private 3-stage ring: one 2-D TMA tile load per
//     64-dim half of K and V (4 x 2 KiB per page, 128-byte swizzle), completion on an mbarrier
//     (bounded waits, no spin without limit);
//   * scores S = K Q^T with tokens as the M dimension and the g query heads of the GQA group
//     as N (mma.sync m16n8k16 bf16 -> fp32); online softmax in the exp2 domain with
//     warp-shuffle column maxima; P^T reaches the PV product through movmatrix.trans; P is
//     split into bf16 hi + lo parts so the PV product keeps ~fp32 accuracy.
// Two kernels:
//   * local set (at most s + w positions per sequence): one thread-block cluster per
//     (sequence, KV head); its CTAs split the pages and merge their partials through
//     distributed shared memory, no global scratch;
//   * full set (flag-gated, up to the whole history): a persistent grid whose CTAs own equal
//     contiguous ranges of (sequence, KV head, page) units enumerated on the device from pos[]
//     and flag[] (unflagged sequences cost nothing, the host never syncs); each range's piece
//     of a (b, h) leaves one partial in global scratch, and the CTA that completes a (b, h)
//     (completion counter, no waiting) merges them with the staged current token.
// Consecutive attention launches of one context may overlap (programmatic dependent launch):
// a launch prefetches its first pages before waiting for the previous one.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cooperative_groups.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace oda {
namespace {

// full set: 4 warps per CTA, two CTAs per SM; local set: 8 warps, one CTA per SM (its
// launch is latency-bound, so more warps in flight beat the room for a second CTA)
constexpr int kW = 4;                 // full set: warps per CTA (each streams its own pages)
constexpr int kThreads = kW * 32;
constexpr int kWL = 8;                // local set: warps per CTA
constexpr int kThreadsL = kWL * 32;
constexpr int kPageTok = 16;
constexpr int kStageBytes = 8192;     // K (4 KiB) + V (4 KiB) of one (page, KV head)
constexpr int kMergeStride = 132;     // floats per (warp, head) row of the merge area
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMaxCluster = 8;
constexpr int kChunk = 4;             // full set: pages per claimed chunk
constexpr int kMergeRows = 20;        // full set: partial rows folded per round of the merge

struct AttnParams {
  const int32_t* page_table;
  const int32_t* pos;
  const int32_t* flag;
  const uint8_t* kv8;     // fp8 pages: blocks [n_pages][Hkv][kF8Block] (unused for bf16 pages)
  const uint32_t* q;      // bf16 pairs [B][Hq][64]
  const uint32_t* k_new;  // bf16 pairs [B][Hkv][64]
  const uint32_t* v_new;
  float* out;             // [B][Hq][128]
  float* part_o;          // full set: [slot][g][128]   slot = CTA index + b*Hkv + h
  float* part_ml;         // full set: [slot][g][2]
  int32_t* counters;      // full set: [B*Hkv] completion counts of the (b, h) partials
  int32_t* claims;        // full set: [B*Hkv] chunk claim counters
  int32_t* err;
  int64_t n_pool_pages;
  int32_t B, Hq, Hkv, g, max_pages, sinks, window, mode;
  int32_t cluster;        // local set: CTAs per (b, h)
  int32_t kv_single;      // 1: tmA spans both pools (one copy per page); 0: tmA = K, tmB = V
  int32_t cta_perm;       // full set: stride of the CTA -> range permutation (coprime to grid)
  int32_t deterministic;  // full set: chunks in a fixed pattern instead of run-time claims
  float scale_log2;       // log2(e) / sqrt(128)
};

// Which cached tokens (0-based indices j < n_cache) a sequence reads, as at most two page
// ranges [0, a_len) and [b_lo, b_lo + b_len) plus a per-token membership test.
struct Geom {
  int active;
  int n_cache;   // cached positions 1..t-1 (token indices 0..t-2)
  int sink_hi;   // local: j < sink_hi is one of the first s positions
  int win_lo;    // local: j >= win_lo is inside the w-window (which also holds t)
  int a_len, b_lo, b_len;
};

__device__ __forceinline__ Geom make_geom(int t, int mode, int sinks, int window, int max_pages,
                                          bool wanted) {
  Geom g;
  g.active = wanted && t >= 1 && (int64_t)(t - 1) <= (int64_t)max_pages * kPageTok;
  g.n_cache = g.active ? t - 1 : 0;
  g.sink_hi = 0;
  g.win_lo = 0;
  g.a_len = 0;
  g.b_lo = 0;
  g.b_len = 0;
  const int n = g.n_cache;
  if (n == 0) return g;
  if (mode == 1) {  // S^F: every cached position
    g.b_len = (n + kPageTok - 1) / kPageTok;
    return g;
  }
  // S^L: positions 1..min(s,t) and max(1, t-w+1)..t  ->  j < min(s, n) or j >= max(0, t-w)
  g.sink_hi = min(sinks, n);
  const long long wl = (long long)t - window;
  g.win_lo = wl > 0 ? (int)wl : 0;
  const int sp = (g.sink_hi + kPageTok - 1) / kPageTok;
  if (g.win_lo >= n) {
    g.a_len = sp;
    return g;
  }
  const int wlo = g.win_lo / kPageTok, whi = (n - 1) / kPageTok;
  if (sp > 0 && wlo <= sp) {
    g.b_len = max(sp, whi + 1);
  } else {
    g.a_len = sp;
    g.b_lo = wlo;
    g.b_len = whi - wlo + 1;
  }
  return g;
}

__device__ __forceinline__ int geom_pages(const Geom& g) { return g.a_len + g.b_len; }

__device__ __forceinline__ int geom_page(const Geom& g, int v) {
  return v < g.a_len ? v : g.b_lo + (v - g.a_len);
}

__device__ __forceinline__ bool geom_has(const Geom& g, int j) {
  return j < g.n_cache && (j < g.sink_hi || j >= g.win_lo);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Online-softmax state of one warp for the g (<= 8) query heads of one KV head.  Lane
// (r = lane/4, c = lane%4) holds heads 2c and 2c+1; o holds O^T fragments (dims x heads).
struct WarpAcc {
  float m0, m1, l0, l1;
  float o[8][4];
  int e;   // fp8 pages: o is held in units of 2^e (the V-scale binade of the last page step)
};

__device__ __forceinline__ void acc_init(WarpAcc& A) {
  A.e = 0;
  A.m0 = A.m1 = -INFINITY;
  A.l0 = A.l1 = 0.f;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) A.o[mt][0] = A.o[mt][1] = A.o[mt][2] = A.o[mt][3] = 0.f;
}

// Query fragments (B operand of S = K Q^T): head n = lane/4 of the group, dims 2c, 2c+1.
__device__ __forceinline__ void load_qf(uint32_t (&qf)[8][2], const AttnParams& p, int b, int h,
                                        int lane) {
  const int n = lane >> 2, c = lane & 3;
  if (n < p.g) {
    const uint32_t* qrow = p.q + ((size_t)b * p.Hq + h * p.g + n) * 64;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qf[kk][0] = qrow[kk * 8 + c];
      qf[kk][1] = qrow[kk * 8 + 4 + c];
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) qf[kk][0] = qf[kk][1] = 0u;
  }
}

// Issues the copy of one (page, KV head) into a stage (K at +0, V at +4096; each as two
// 64-column halves of 16 rows, 128-byte swizzle): one 4-D copy when a single map spans both
// pools, else one 3-D copy per pool.
__device__ __forceinline__ void issue_page(uint8_t* dst, uint64_t* bar, const CUtensorMap* tmA,
                                           const CUtensorMap* tmB, bool single, int phys, int Hkv,
                                           int h) {
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(bar, kStageBytes);
  const int y = (phys * Hkv + h) * kPageTok;
  if (single) {
    tma_load_4d(dst, tmA, 0, y, 0, 0, bar);
  } else {
    tma_load_3d(dst, tmA, 0, y, 0, bar);
    tma_load_3d(dst + 4096, tmB, 0, y, 0, bar);
  }
}

// One 16-token page in a stage: scores, online softmax, PV.  in0 / in1: whether this lane's
// token rows r and r + 8 belong to the set.  Warp-uniform; no-op if no token belongs.
__device__ __forceinline__ void page_compute(WarpAcc& A, const uint32_t (&qf)[8][2],
                                             uint8_t* stage, bool in0, bool in1,
                                             float scale_log2, int lane) {
  if (!__any_sync(0xffffffffu, in0 || in1)) return;
  const int r = lane >> 2, c = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;     // ldmatrix: matrix index, row in matrix
  const int krow = ((mi & 1) << 3) + rr;       // K tile row (token) this lane addresses
  const int vrow = ((mi >> 1) << 3) + rr;      // V tile row (token) this lane addresses
  const uint32_t sb = smem_u32(stage);
  // S[token][head] = K[token] . Q[head]; two independent accumulation chains
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < 8; kk += 2) {
    uint32_t a0[4], a1[4];
    const int ch0 = 2 * kk + (mi >> 1), ch1 = ch0 + 2;
    ldsm_x4(a0, sb + (ch0 >> 3) * 2048 + krow * 128 + (((ch0 & 7) ^ rr) << 4));
    ldsm_x4(a1, sb + (ch1 >> 3) * 2048 + krow * 128 + (((ch1 & 7) ^ rr) << 4));
    mma_bf16_16816(sa, a0, qf[kk][0], qf[kk][1]);
    mma_bf16_16816(sb2, a1, qf[kk + 1][0], qf[kk + 1][1]);
  }
  const float x0 = in0 ? (sa[0] + sb2[0]) * scale_log2 : -INFINITY;
  const float x1 = in0 ? (sa[1] + sb2[1]) * scale_log2 : -INFINITY;
  const float x2 = in1 ? (sa[2] + sb2[2]) * scale_log2 : -INFINITY;
  const float x3 = in1 ? (sa[3] + sb2[3]) * scale_log2 : -INFINITY;
  float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = fmaxf(A.m0, mx0), mn1 = fmaxf(A.m1, mx1);
  if (mn0 > A.m0 || mn1 > A.m1) {
    const float al0 = exp2f(A.m0 - mn0), al1 = exp2f(A.m1 - mn1);
    A.l0 *= al0;
    A.l1 *= al1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      A.o[mt][0] *= al0;
      A.o[mt][1] *= al1;
      A.o[mt][2] *= al0;
      A.o[mt][3] *= al1;
    }
    A.m0 = mn0;
    A.m1 = mn1;
  }
  const float p0 = exp2f(x0 - A.m0), p1 = exp2f(x1 - A.m1);
  const float p2 = exp2f(x2 - A.m0), p3 = exp2f(x3 - A.m1);
  A.l0 += p0 + p2;
  A.l1 += p1 + p3;
  const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
  const __nv_bfloat16 h2 = __float2bfloat16_rn(p2), h3 = __float2bfloat16_rn(p3);
  const uint32_t hi01 = pack_bf16x2(h0, h1), hi23 = pack_bf16x2(h2, h3);
  const uint32_t lo01 = pack_bf16x2(__float2bfloat16_rn(p0 - __bfloat162float(h0)),
                                    __float2bfloat16_rn(p1 - __bfloat162float(h1)));
  const uint32_t lo23 = pack_bf16x2(__float2bfloat16_rn(p2 - __bfloat162float(h2)),
                                    __float2bfloat16_rn(p3 - __bfloat162float(h3)));
  // P^T fragments (k = token, n = head) for the PV product
  const uint32_t bh0 = movmatrix_trans(hi01), bh1 = movmatrix_trans(hi23);
  const uint32_t bl0 = movmatrix_trans(lo01), bl1 = movmatrix_trans(lo23);
  // Tokens outside the set have P = 0, but their V rows may hold stale bytes (slots not yet
  // committed, or a partly filled page): 0 * NaN would poison the sum, so zero them.
  if (__any_sync(0xffffffffu, !(in0 && in1))) {
    uint4* vbase = reinterpret_cast<uint4*>(stage + 4096);
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    if (!in0) {   // token row r: 8 x 16 bytes in each 64-dim half
      vbase[r * 8 + 2 * c] = z;
      vbase[r * 8 + 2 * c + 1] = z;
      vbase[128 + r * 8 + 2 * c] = z;
      vbase[128 + r * 8 + 2 * c + 1] = z;
    }
    if (!in1) {   // token row r + 8
      vbase[(r + 8) * 8 + 2 * c] = z;
      vbase[(r + 8) * 8 + 2 * c + 1] = z;
      vbase[128 + (r + 8) * 8 + 2 * c] = z;
      vbase[128 + (r + 8) * 8 + 2 * c + 1] = z;
    }
    __syncwarp();
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int chunk = 2 * mt + (mi & 1);
    uint32_t a[4];
    ldsm_x4_trans(a, sb + 4096 + (chunk >> 3) * 2048 + vrow * 128 + (((chunk & 7) ^ rr) << 4));
    mma_bf16_16816(A.o[mt], a, bh0, bh1);
    mma_bf16_16816(A.o[mt], a, bl0, bl1);
  }
}

// Scores S = K Q^T of one 16-token page (tokens as M, the group's heads as N), in the exp2
// domain; tokens outside the set get -inf.
__device__ __forceinline__ void page_scores(float (&x)[4], const uint32_t (&qf)[8][2], uint32_t sb,
                                            bool in0, bool in1, float scale_log2, int lane) {
  const int mi = lane >> 3, rr = lane & 7;
  const int krow = ((mi & 1) << 3) + rr;
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < 8; kk += 2) {
    uint32_t a0[4], a1[4];
    const int ch0 = 2 * kk + (mi >> 1), ch1 = ch0 + 2;
    ldsm_x4(a0, sb + (ch0 >> 3) * 2048 + krow * 128 + (((ch0 & 7) ^ rr) << 4));
    ldsm_x4(a1, sb + (ch1 >> 3) * 2048 + krow * 128 + (((ch1 & 7) ^ rr) << 4));
    mma_bf16_16816(sa, a0, qf[kk][0], qf[kk][1]);
    mma_bf16_16816(sc, a1, qf[kk + 1][0], qf[kk + 1][1]);
  }
  x[0] = in0 ? (sa[0] + sc[0]) * scale_log2 : -INFINITY;
  x[1] = in0 ? (sa[1] + sc[1]) * scale_log2 : -INFINITY;
  x[2] = in1 ? (sa[2] + sc[2]) * scale_log2 : -INFINITY;
  x[3] = in1 ? (sa[3] + sc[3]) * scale_log2 : -INFINITY;
}

// P (fp32, this lane's rows r / r + 8 and heads 2c / 2c + 1) as P^T fragments for the PV
// product, split into bf16 hi + lo parts.
__device__ __forceinline__ void p_fragments(const float (&pv)[4], uint32_t& bh0, uint32_t& bh1,
                                            uint32_t& bl0, uint32_t& bl1) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(pv[0]), h1 = __float2bfloat16_rn(pv[1]);
  const __nv_bfloat16 h2 = __float2bfloat16_rn(pv[2]), h3 = __float2bfloat16_rn(pv[3]);
  bh0 = movmatrix_trans(pack_bf16x2(h0, h1));
  bh1 = movmatrix_trans(pack_bf16x2(h2, h3));
  bl0 = movmatrix_trans(pack_bf16x2(__float2bfloat16_rn(pv[0] - __bfloat162float(h0)),
                                    __float2bfloat16_rn(pv[1] - __bfloat162float(h1))));
  bl1 = movmatrix_trans(pack_bf16x2(__float2bfloat16_rn(pv[2] - __bfloat162float(h2)),
                                    __float2bfloat16_rn(pv[3] - __bfloat162float(h3))));
}

// Zeroes the V rows of tokens outside the set (their P is 0, but stale bytes could be NaN).
// Returns true if it wrote to the stage.
__device__ __forceinline__ bool zero_masked_v(uint8_t* stage, bool in0, bool in1, int lane) {
  if (!__any_sync(0xffffffffu, !(in0 && in1))) return false;
  const int r = lane >> 2, c = lane & 3;
  uint4* vbase = reinterpret_cast<uint4*>(stage + 4096);
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  if (!in0) {
    vbase[r * 8 + 2 * c] = z;
    vbase[r * 8 + 2 * c + 1] = z;
    vbase[128 + r * 8 + 2 * c] = z;
    vbase[128 + r * 8 + 2 * c + 1] = z;
  }
  if (!in1) {
    vbase[(r + 8) * 8 + 2 * c] = z;
    vbase[(r + 8) * 8 + 2 * c + 1] = z;
    vbase[128 + (r + 8) * 8 + 2 * c] = z;
    vbase[128 + (r + 8) * 8 + 2 * c + 1] = z;
  }
  __syncwarp();
  return true;
}

// Two pages (32 tokens) in one online-softmax step: both score blocks are independent, the
// running maximum and the rescale are taken once for the pair, and the PV products of the two
// pages accumulate into separate hi / lo chains.  Same result as two page_compute calls up to
// fp32 rounding.
__device__ __forceinline__ void page_compute2(WarpAcc& A, const uint32_t (&qf)[8][2],
                                              uint8_t* stA, bool a0, bool a1,
                                              uint8_t* stB, bool b0, bool b1,
                                              float scale_log2, int lane) {
  const bool anyA = __any_sync(0xffffffffu, a0 || a1), anyB = __any_sync(0xffffffffu, b0 || b1);
  if (!anyA || !anyB) {   // a page without tokens in the set: the other one alone
    if (anyA) page_compute(A, qf, stA, a0, a1, scale_log2, lane);
    if (anyB) page_compute(A, qf, stB, b0, b1, scale_log2, lane);
    return;
  }
  const int mi = lane >> 3, rr = lane & 7;
  const int vrow = ((mi >> 1) << 3) + rr;
  const uint32_t sA = smem_u32(stA), sB = smem_u32(stB);
  float xa[4], xb[4];
  page_scores(xa, qf, sA, a0, a1, scale_log2, lane);
  page_scores(xb, qf, sB, b0, b1, scale_log2, lane);
  float mx0 = fmaxf(fmaxf(xa[0], xa[2]), fmaxf(xb[0], xb[2]));
  float mx1 = fmaxf(fmaxf(xa[1], xa[3]), fmaxf(xb[1], xb[3]));
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = fmaxf(A.m0, mx0), mn1 = fmaxf(A.m1, mx1);
  if (mn0 > A.m0 || mn1 > A.m1) {
    const float al0 = exp2f(A.m0 - mn0), al1 = exp2f(A.m1 - mn1);
    A.l0 *= al0;
    A.l1 *= al1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      A.o[mt][0] *= al0;
      A.o[mt][1] *= al1;
      A.o[mt][2] *= al0;
      A.o[mt][3] *= al1;
    }
    A.m0 = mn0;
    A.m1 = mn1;
  }
  float pa[4], pb[4];
  pa[0] = exp2f(xa[0] - A.m0);
  pa[1] = exp2f(xa[1] - A.m1);
  pa[2] = exp2f(xa[2] - A.m0);
  pa[3] = exp2f(xa[3] - A.m1);
  pb[0] = exp2f(xb[0] - A.m0);
  pb[1] = exp2f(xb[1] - A.m1);
  pb[2] = exp2f(xb[2] - A.m0);
  pb[3] = exp2f(xb[3] - A.m1);
  A.l0 += (pa[0] + pa[2]) + (pb[0] + pb[2]);
  A.l1 += (pa[1] + pa[3]) + (pb[1] + pb[3]);
  uint32_t ah0, ah1, al0, al1, bh0, bh1, bl0, bl1;
  p_fragments(pa, ah0, ah1, al0, al1);
  p_fragments(pb, bh0, bh1, bl0, bl1);
  zero_masked_v(stA, a0, a1, lane);
  zero_masked_v(stB, b0, b1, lane);
  float lo[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) lo[mt][0] = lo[mt][1] = lo[mt][2] = lo[mt][3] = 0.f;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int chunk = 2 * mt + (mi & 1);
    const uint32_t off = 4096 + (chunk >> 3) * 2048 + vrow * 128 + (((chunk & 7) ^ rr) << 4);
    uint32_t va[4], vb[4];
    ldsm_x4_trans(va, sA + off);
    ldsm_x4_trans(vb, sB + off);
    mma_bf16_16816(A.o[mt], va, ah0, ah1);
    mma_bf16_16816(lo[mt], va, al0, al1);
    mma_bf16_16816(A.o[mt], vb, bh0, bh1);
    mma_bf16_16816(lo[mt], vb, bl0, bl1);
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    A.o[mt][0] += lo[mt][0];
    A.o[mt][1] += lo[mt][1];
    A.o[mt][2] += lo[mt][2];
    A.o[mt][3] += lo[mt][3];
  }
}

// ------------------------------------------------------------------ fp8 (e4m3) pages
// One (page, KV head) block of an fp8 pool is kF8Block contiguous bytes, brought in by one bulk
// copy:
//   [0, 2048)     K codes, token-major: token j's 128 codes at 128*j, its 16-dim chunk k stored
//                 at chunk position k ^ (j & 7) (so ldmatrix rows of 8 tokens hit 8 bank groups);
//   [2048, 4096)  V codes transposed: dim d's 16 codes at 2048 + 16*d, slot s holding token
//                 tau(s) = 2*(s/4) + (s&1) + 8*((s>>1)&1), i.e. slots 4c..4c+3 hold tokens
//                 2c, 2c+1, 2c+8, 2c+9 (the token order of a P^T fragment);
//   [4096, 4160)  K scales, fp32 [16], token order;  [4160, 4224)  V scales, fp32 [16].
// Cached value = scale * e4m3 value of its code.  The codes convert exactly to f16 for the
// tensor-core products; the K scale multiplies each token's score after the QK^T product; the
// V scale multiplies each token's probability before the PV product (normalised per page by a
// power of two that is multiplied back into the accumulator, so f16 keeps its range).
constexpr int kF8Block = 4224;
constexpr int kF8V = 2048;
constexpr int kF8SK = 4096;
constexpr int kF8SV = 4160;

// q of one KV head's group as f16 B fragments in the fp8 dimension order, scaled per head by a
// power of two 2^e_n (max |q_n| * 2^e_n in [2^14, 2^15)); fs0 / fs1 undo it (times log2(e)/sqrt(d))
// for the heads 2c, 2c + 1 of this lane's score columns.
struct QF8 {
  uint32_t qf[8][2];
  float fs0, fs1;
};

__device__ __forceinline__ void load_q8(QF8& Q, const AttnParams& p, int b, int h, int lane) {
  const int n = lane >> 2, c = lane & 3;
  float v[8][4];
  float mx = 0.f;
  if (n < p.g) {
    const uint32_t* qrow = p.q + ((size_t)b * p.Hq + h * p.g + n) * 64;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t w0 = qrow[8 * kk + 2 * c], w1 = qrow[8 * kk + 2 * c + 1];
      v[kk][0] = bf16_lo_to_f32(w0);
      v[kk][1] = bf16_hi_to_f32(w0);
      v[kk][2] = bf16_lo_to_f32(w1);
      v[kk][3] = bf16_hi_to_f32(w1);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v[kk][0]), fabsf(v[kk][1])), fmaxf(fabsf(v[kk][2]), fabsf(v[kk][3]))));
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) v[kk][0] = v[kk][1] = v[kk][2] = v[kk][3] = 0.f;
  }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  int e = 0;
  if (mx > 0.f && mx <= 3.0e38f) {
    const int ex = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127;   // floor(log2(mx)), normal mx
    e = min(60, max(-60, 14 - ex));
  }
  const float up = __uint_as_float((uint32_t)(127 + e) << 23);
  const float down = (n < p.g) ? p.scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23) : 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    Q.qf[kk][0] = pack_f16x2(v[kk][0] * up, v[kk][1] * up);
    Q.qf[kk][1] = pack_f16x2(v[kk][2] * up, v[kk][3] * up);
  }
  Q.fs0 = __shfl_sync(0xffffffffu, down, 8 * c);
  Q.fs1 = __shfl_sync(0xffffffffu, down, 8 * c + 4);
}

// K fragments of one fp8 page (tokens as M in natural order, dims in the q fragment order) and
// V^T fragments (dims as M, tokens in the P^T fragment order), converted to f16.
// Raw scores K q^T of one fp8 page (tokens as M in natural order, dims in the q fragment
// order), before scales: K fragments by ldmatrix, converted to f16 from the register halves.
__device__ __forceinline__ void page_scores8(float (&sacc)[4], const QF8& Q, uint32_t sb, int lane) {
  const int mi = lane >> 3, rr = lane & 7;
  const int tok = ((mi & 1) << 3) + rr;          // token row this lane addresses
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < 8; kk += 2) {
    uint32_t r[4], a0[4], a1[4];
    ldsm_x4(r, sb + tok * 128 + (((kk + (mi >> 1)) ^ rr) << 4));
    e4m3x4_to_f16x2x2(r[0], a0[0], a0[2]);
    e4m3x4_to_f16x2x2(r[1], a0[1], a0[3]);
    e4m3x4_to_f16x2x2(r[2], a1[0], a1[2]);
    e4m3x4_to_f16x2x2(r[3], a1[1], a1[3]);
    mma_f16_16816(sa, a0, Q.qf[kk][0], Q.qf[kk][1]);
    mma_f16_16816(sc, a1, Q.qf[kk + 1][0], Q.qf[kk + 1][1]);
  }
  sacc[0] = sa[0] + sc[0];
  sacc[1] = sa[1] + sc[1];
  sacc[2] = sa[2] + sc[2];
  sacc[3] = sa[3] + sc[3];
}

// PV of one fp8 page into the accumulator: V^T fragments (dims as M, tokens in the P^T fragment
// order) by ldmatrix, converted to f16, masked where tokens are outside the set.
__device__ __forceinline__ void page_pv8(float (&o)[8][4], uint32_t vb, uint32_t bh0, uint32_t bh1,
                                         uint32_t bl0, uint32_t bl1, bool masked, uint32_t mlo,
                                         uint32_t mhi, int lane) {
  const int mi = lane >> 3, rr = lane & 7;
  const int drow = ((mi & 1) << 3) + rr;         // dim row within a 16-dim tile
#pragma unroll
  for (int mt = 0; mt < 8; mt += 2) {
    uint32_t r[4], a0[4], a1[4];
    ldsm_x4(r, vb + (16 * (mt + (mi >> 1)) + drow) * 16);
    e4m3x4_to_f16x2x2(r[0], a0[0], a0[2]);
    e4m3x4_to_f16x2x2(r[1], a0[1], a0[3]);
    e4m3x4_to_f16x2x2(r[2], a1[0], a1[2]);
    e4m3x4_to_f16x2x2(r[3], a1[1], a1[3]);
    if (masked) {   // tokens outside the set: their codes may be stale (even NaN); P'' is 0 there
      a0[0] &= mlo; a0[1] &= mlo; a0[2] &= mhi; a0[3] &= mhi;
      a1[0] &= mlo; a1[1] &= mlo; a1[2] &= mhi; a1[3] &= mhi;
    }
    mma_f16_16816(o[mt], a0, bh0, bh1);
    mma_f16_16816(o[mt], a0, bl0, bl1);
    mma_f16_16816(o[mt + 1], a1, bh0, bh1);
    mma_f16_16816(o[mt + 1], a1, bl0, bl1);
  }
}

// Keep-masks of this lane's V^T fragment halves for a page whose token set is given by the
// lanes' (in0, in1): the low word of a fragment holds tokens 2c, 2c+1, the high word 2c+8, 2c+9.
__device__ __forceinline__ void v8_masks(bool in0, bool in1, int lane, uint32_t& mlo, uint32_t& mhi) {
  auto squeeze = [](uint32_t x) {   // bits 0, 4, ..., 28 -> bits 0..7
    x &= 0x11111111u;
    x = (x | (x >> 3)) & 0x03030303u;
    x = (x | (x >> 6)) & 0x000F000Fu;
    return (x | (x >> 12)) & 0xFFu;
  };
  const uint32_t t_lo = squeeze(__ballot_sync(0xffffffffu, in0));   // tokens 0..7
  const uint32_t t_hi = squeeze(__ballot_sync(0xffffffffu, in1));   // tokens 8..15
  const int c = lane & 3;
  const uint32_t a = (t_lo >> (2 * c)) & 3u, bb = (t_hi >> (2 * c)) & 3u;
  mlo = ((a & 1u) ? 0x0000FFFFu : 0u) | ((a & 2u) ? 0xFFFF0000u : 0u);
  mhi = ((bb & 1u) ? 0x0000FFFFu : 0u) | ((bb & 2u) ? 0xFFFF0000u : 0u);
}

// NP (1 or 2) fp8 pages in one online-softmax step (one maximum and rescale for 16 * NP tokens).
// in[i][0] / in[i][1]: whether this lane's token rows r and r + 8 of page i belong to the set.
// The accumulator is kept in units of 2^A.e, the binade of the largest V scale of the step's
// tokens, so P'' = p * sv * 2^-e stays below 2 and f16 keeps its precision; when the binade
// changes the accumulator is rescaled by the (exact) power of two, together with the softmax's
// own rescale.
template <int NP>
__device__ __forceinline__ void page_step8(WarpAcc& A, const QF8& Q, uint8_t* const (&st)[2],
                                           const bool (&in)[2][2], int lane) {
  const int r = lane >> 2;
  float x[2][4], svv[2][2];
  bool any_masked = false;
  float svmax = 0.f;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    float sacc[4];
    page_scores8(sacc, Q, smem_u32(st[i]), lane);
    const float* sk = reinterpret_cast<const float*>(st[i] + kF8SK);
    const float* sv = reinterpret_cast<const float*>(st[i] + kF8SV);
    const float k0 = sk[r], k1 = sk[r + 8];
    x[i][0] = in[i][0] ? sacc[0] * k0 * Q.fs0 : -INFINITY;
    x[i][1] = in[i][0] ? sacc[1] * k0 * Q.fs1 : -INFINITY;
    x[i][2] = in[i][1] ? sacc[2] * k1 * Q.fs0 : -INFINITY;
    x[i][3] = in[i][1] ? sacc[3] * k1 * Q.fs1 : -INFINITY;
    svv[i][0] = in[i][0] ? sv[r] : 0.f;
    svv[i][1] = in[i][1] ? sv[r + 8] : 0.f;
    svmax = fmaxf(svmax, fmaxf(svv[i][0], svv[i][1]));
    any_masked |= !(in[i][0] && in[i][1]);
  }
  float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
  if (NP == 2) {
    mx0 = fmaxf(mx0, fmaxf(x[1][0], x[1][2]));
    mx1 = fmaxf(mx1, fmaxf(x[1][1], x[1][3]));
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    svmax = fmaxf(svmax, __shfl_xor_sync(0xffffffffu, svmax, off));
  }
  const int E = (svmax > 0.f && svmax <= 3.0e38f)
                    ? min(126, max(-126, (int)((__float_as_uint(svmax) >> 23) & 0xFF) - 127))
                    : A.e;
  const float down = __uint_as_float((uint32_t)(127 - E) << 23);
  const float mn0 = fmaxf(A.m0, mx0), mn1 = fmaxf(A.m1, mx1);
  if (mn0 > A.m0 || mn1 > A.m1 || E != A.e) {
    // o in units of 2^A.e -> units of 2^E, with the softmax rescale; -inf maxima give 0
    const float al0 = exp2f(A.m0 - mn0), al1 = exp2f(A.m1 - mn1);
    A.l0 *= al0;
    A.l1 *= al1;
    const float f0 = ldexpf(al0, A.e - E), f1 = ldexpf(al1, A.e - E);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      A.o[mt][0] *= f0;
      A.o[mt][1] *= f1;
      A.o[mt][2] *= f0;
      A.o[mt][3] *= f1;
    }
    A.m0 = mn0;
    A.m1 = mn1;
    A.e = E;
  }
  const bool masked = __any_sync(0xffffffffu, any_masked);
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const float p0 = exp2f(x[i][0] - A.m0), p1 = exp2f(x[i][1] - A.m1);
    const float p2 = exp2f(x[i][2] - A.m0), p3 = exp2f(x[i][3] - A.m1);
    A.l0 += p0 + p2;
    A.l1 += p1 + p3;
    const float s0 = svv[i][0] * down, s1 = svv[i][1] * down;
    const float q0 = p0 * s0, q1 = p1 * s0, q2 = p2 * s1, q3 = p3 * s1;
    const uint32_t h01 = pack_f16x2(q0, q1), h23 = pack_f16x2(q2, q3);
    const uint32_t l01 = pack_f16x2(q0 - f16_lo_to_f32(h01), q1 - f16_hi_to_f32(h01));
    const uint32_t l23 = pack_f16x2(q2 - f16_lo_to_f32(h23), q3 - f16_hi_to_f32(h23));
    const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
    const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);
    uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
    if (masked) v8_masks(in[i][0], in[i][1], lane, mlo, mhi);
    page_pv8(A.o, smem_u32(st[i] + kF8V), bh0, bh1, bl0, bl1, masked, mlo, mhi, lane);
  }
}

// Issues the bulk copy of one fp8 (page, KV head) block into a stage.
__device__ __forceinline__ void issue_page8(uint8_t* dst, uint64_t* bar, const uint8_t* kv8,
                                            int phys, int Hkv, int h) {
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(bar, kF8Block);
  bulk_load(dst, kv8 + ((size_t)phys * Hkv + h) * kF8Block, kF8Block, bar);
}

// Reduces l over the token rows and writes the warp's state to its merge slot:
// mo [g][kMergeStride] (O^T columns), ml [8][2] (m, l).
__device__ __forceinline__ void warp_flush(WarpAcc& A, float* mo, float* ml, int g, int lane) {
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    A.l0 += __shfl_xor_sync(0xffffffffu, A.l0, off);
    A.l1 += __shfl_xor_sync(0xffffffffu, A.l1, off);
  }
  if (A.e != 0) {   // warp-uniform
    const float u = __uint_as_float((uint32_t)(127 + A.e) << 23);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      A.o[mt][0] *= u;
      A.o[mt][1] *= u;
      A.o[mt][2] *= u;
      A.o[mt][3] *= u;
    }
    A.e = 0;
  }
  const int r = lane >> 2, c = lane & 3;
  const int n0 = 2 * c, n1 = 2 * c + 1;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d = 16 * mt + r;
    if (n0 < g) {
      mo[n0 * kMergeStride + d] = A.o[mt][0];
      mo[n0 * kMergeStride + d + 8] = A.o[mt][2];
    }
    if (n1 < g) {
      mo[n1 * kMergeStride + d] = A.o[mt][1];
      mo[n1 * kMergeStride + d + 8] = A.o[mt][3];
    }
  }
  if (r == 0) {
    ml[n0 * 2] = A.m0;
    ml[n0 * 2 + 1] = A.l0;
    ml[n1 * 2] = A.m1;
    ml[n1 * 2 + 1] = A.l1;
  }
}

// Merge of the W warp states for head n, dim d: (M, L, O) relative to exp2(M).
template <int W>
__device__ __forceinline__ void cta_merge(const float* merge_o, const float* merge_ml, int g,
                                          int n, int d, float& M, float& L, float& O) {
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < W; ++w) M = fmaxf(M, merge_ml[w * 16 + n * 2]);
  O = 0.f;
  L = 0.f;
  if (M == -INFINITY) return;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const float mw = merge_ml[w * 16 + n * 2];
    if (mw != -INFINITY) {
      const float sc = exp2f(mw - M);
      O += sc * merge_o[(w * g + n) * kMergeStride + d];
      L += sc * merge_ml[w * 16 + n * 2 + 1];
    }
  }
}

__device__ __forceinline__ float staged_value(const AttnParams& p, int b, int h, int d) {
  const uint32_t vv = p.v_new[((size_t)b * p.Hkv + h) * 64 + (d >> 1)];
  return (d & 1) ? bf16_hi_to_f32(vv) : bf16_lo_to_f32(vv);
}

// Work units are (sequence b, KV head h, visited page v) in (b, h, v) order; every active
// sequence has max(1, pages) units per KV head (an empty cache keeps one unit that loads
// nothing, so the staged token still produces the output).  CTA c owns the contiguous unit
// range [c*U/G, (c+1)*U/G) with G = min(grid size, U): equal work per CTA.  The part of that range inside one (b, h)
// is a segment; each segment yields one partial in slot c + b*Hkv + h (unique, since the
// CTAs walk the (b, h) pairs in order).
struct Seg {
  int b, h, v0, n;   // first visited page of the segment, units in this CTA's segment
  int s0, nv;        // first unit of (b, h) and units per KV head of sequence b
};

__device__ __forceinline__ Seg decode_seg(int u, int u1, const int* s_us, const int* s_nv, int B,
                                          int Hkv) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_us[mid] <= u) lo = mid; else hi = mid - 1;
  }
  Seg s;
  s.b = lo;
  s.nv = s_nv[lo];
  const int r = u - s_us[lo];
  s.h = r / s.nv;
  s.v0 = r - s.h * s.nv;
  s.s0 = s_us[lo] + s.h * s.nv;
  s.n = min(u1, s.s0 + s.nv) - u;
  return s;
}

// CTA owning unit u when G CTAs split U units.
__device__ __forceinline__ int cta_of(long long u, long long U, long long G) {
  return (int)(((u + 1) * G - 1) / U);
}

// Page formats: F = 0 bf16 pools (one 4-D / two 3-D TMA tile copies of 8 KiB per page),
// F = 1 fp8 blocks (one bulk copy of kF8Block bytes).  The fp8 stages are about half the size,
// so the rings hold twice as many pages and the bytes in flight stay the same.
template <int F> struct Fmt;
template <> struct Fmt<0> {
  static constexpr int kStage = kStageBytes, kR = 3, kRL = 3, kAlign = 1024, kMinCtas = 2;
};
template <> struct Fmt<1> {
  static constexpr int kStage = kF8Block, kR = 3, kRL = 6, kAlign = 128, kMinCtas = 3;
};

// Query fragments of either format.
template <int F> struct QFrag;
template <> struct QFrag<0> { uint32_t qf[8][2]; };
template <> struct QFrag<1> { QF8 q; };

template <int F>
__device__ __forceinline__ void load_q(QFrag<F>& Q, const AttnParams& p, int b, int h, int lane) {
  if constexpr (F == 0) load_qf(Q.qf, p, b, h, lane);
  else load_q8(Q.q, p, b, h, lane);
}

template <int F>
__device__ __forceinline__ void issue_any(uint8_t* dst, uint64_t* bar, const CUtensorMap* tmA,
                                          const CUtensorMap* tmB, const AttnParams& p, int phys, int h) {
  if constexpr (F == 0) issue_page(dst, bar, tmA, tmB, p.kv_single, phys, p.Hkv, h);
  else issue_page8(dst, bar, p.kv8, phys, p.Hkv, h);
}

// One page (a1 = a0 = false for b: single) or two pages in one online-softmax step.
template <int F>
__device__ __forceinline__ void pages_compute(WarpAcc& A, const QFrag<F>& Q, uint8_t* stA, bool a0,
                                              bool a1, uint8_t* stB, bool b0, bool b1, bool pair,
                                              float scale_log2, int lane) {
  if constexpr (F == 0) {
    if (pair) page_compute2(A, Q.qf, stA, a0, a1, stB, b0, b1, scale_log2, lane);
    else page_compute(A, Q.qf, stA, a0, a1, scale_log2, lane);
  } else {
    uint8_t* const st[2] = {stA, stB};
    const bool in[2][2] = {{a0, a1}, {b0, b1}};
    const bool anyA = __any_sync(0xffffffffu, a0 || a1);
    const bool anyB = pair && __any_sync(0xffffffffu, b0 || b1);
    if (anyA && anyB) {
      page_step8<2>(A, Q.q, st, in, lane);
    } else if (anyA) {
      page_step8<1>(A, Q.q, st, in, lane);
    } else if (anyB) {
      uint8_t* const stb[2] = {stB, stB};
      const bool inb[2][2] = {{b0, b1}, {b0, b1}};
      page_step8<1>(A, Q.q, stb, inb, lane);
    }
  }
}

// ---------------------------------------------------------------- local set: clusters
// Cluster of p.cluster CTAs per (b, h); CTA `rank` takes the contiguous share
// [rank*nv/C, (rank+1)*nv/C) of the visited pages; warps take every kWL-th page of it.  Each
// rank merges its warps' partials and writes the result straight into rank 0's inbox (distributed
// shared memory), then arrives on rank 0's inbox barrier and exits; rank 0 waits for the C - 1
// arrivals and finishes all g*128 outputs with the staged token.  Nothing but rank 0 waits on
// another CTA after the pages, and no CTA reads another's shared memory.
template <int F>
__global__ void __launch_bounds__(kThreadsL, 1)
attn_local_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const AttnParams p) {
  constexpr int kRL = Fmt<F>::kRL;
  constexpr int kStg = Fmt<F>::kStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + (Fmt<F>::kAlign - 1)) & ~uintptr_t(Fmt<F>::kAlign - 1));
  const int g = p.g;
  // the merge areas reuse the stages: they are written only after every copy has landed
  float* merge_o = reinterpret_cast<float*>(stages);                   // [W][g][132]
  float* merge_ml = merge_o + kWL * g * kMergeStride;                  // [W][8][2]
  // rank 0's inbox (its own region, past the stages: other ranks write it while rank 0 may
  // still stream pages): the ranks' CTA partials o [C][g][128], then (m, l) [C][g][2]
  float* inbox_o = reinterpret_cast<float*>(stages + kWL * kRL * kStg);
  float* inbox_ml = inbox_o + (size_t)p.cluster * g * 128;
  __shared__ __align__(8) uint64_t bars[kWL * kRL];
  __shared__ __align__(8) uint64_t inbox_bar;

  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.cluster;
  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.x / C;
  const int b = bh / p.Hkv, h = bh - (bh / p.Hkv) * p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kWL * kRL; ++i) mbar_init(&bars[i], 1);
    mbar_init(&inbox_bar, C > 1 ? C - 1 : 1);
    fence_mbar_init();
    if (F == 0) {
      prefetch_tensormap(&tmA);
      if (!p.kv_single) prefetch_tensormap(&tmB);
    }
  }
  const int t = __ldcg(p.pos + b);
  const Geom ge = make_geom(t, 0, p.sinks, p.window, p.max_pages, true);
  if (!ge.active && rank == 0 && tid == 0) atomicOr(p.err, ODA_DEVERR_POS_RANGE);
  const int nv = ge.active ? geom_pages(ge) : 0;
  const int v_lo = (int)((long long)rank * nv / C), v_hi = (int)((long long)(rank + 1) * nv / C);
  const int cw = (v_hi - v_lo - warp > 0) ? (v_hi - v_lo - warp + kWL - 1) / kWL : 0;
  const int* ptab = p.page_table + (size_t)b * p.max_pages;
  uint8_t* my_stages = stages + warp * kRL * kStg;
  uint64_t* my_bars = bars + warp * kRL;
  __syncthreads();
  // rank 0's inbox barrier is initialised before any rank arrives on it: every thread arrives
  // here and waits (long after) before the merge
  cluster_arrive();

  // lane k holds the physical page of this warp's (pt_base + k)-th page
  int pt_phys = -1, pt_base = -64;
  auto refill = [&](int base) {
    const int k = base + lane;
    pt_phys = -1;
    if (k < cw && ge.n_cache > 0) {
      const int phys = __ldcg(ptab + geom_page(ge, v_lo + warp + k * kWL));
      pt_phys = (phys >= 0 && (int64_t)phys < p.n_pool_pages) ? phys : -2;
      if (pt_phys == -2) atomicOr(p.err, ODA_DEVERR_PAGE_RANGE);
    }
    pt_base = base;
  };
  uint32_t vbits = 0;
  auto issue = [&](int k) {
    if (k - pt_base >= 32) refill(k & ~31);
    const uint32_t st = (uint32_t)k % kRL;
    const int phys = __shfl_sync(0xffffffffu, pt_phys, k - pt_base);
    if (lane == k - pt_base) {
      if (phys >= 0)
        issue_any<F>(my_stages + st * kStg, my_bars + st, &tmA, &tmB, p, phys, h);
      else
        mbar_arrive(my_bars + st);
    }
    vbits = phys >= 0 ? (vbits | (1u << st)) : (vbits & ~(1u << st));
  };
  for (int k = 0; k < kRL && k < cw; ++k) issue(k);
  // the previous launch on the stream may still run: wait before reading q or writing
  grid_dependency_wait();
  grid_dependents_launch();

  QFrag<F> qf;
  load_q<F>(qf, p, b, h, lane);
  // staged current token: its q . k words (heads warp, warp + kWL) and the value this thread
  // combines first are loaded now and used after the page loop, off the critical path
  __shared__ float s_snew[8];
  uint32_t sq[2][2] = {{0u, 0u}, {0u, 0u}};
  const uint32_t* krow_new = p.k_new + ((size_t)b * p.Hkv + h) * 64;
  const uint32_t sk0 = krow_new[lane], sk1 = krow_new[lane + 32];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int n = warp + i * kWL;
    if (n < g) {
      const uint32_t* qrow = p.q + ((size_t)b * p.Hq + h * g + n) * 64;
      sq[i][0] = qrow[lane];
      sq[i][1] = qrow[lane + 32];
    }
  }
  // rank 0 finishes outputs tid, tid + 256, ... (at most 4 for g <= 8): their staged values now
  float v_staged[(8 * 128) / kThreadsL];
#pragma unroll
  for (int i = 0; i < (8 * 128) / kThreadsL; ++i)
    v_staged[i] = (rank == 0 && tid + i * kThreadsL < g * 128) ? staged_value(p, b, h, (tid + i * kThreadsL) & 127) : 0.f;
  WarpAcc A;
  acc_init(A);
  const int r = lane >> 2;
  int k = 0;
  bool dead = false;
  // pages are taken two at a time (one softmax step for 32 tokens), in fixed pairs so that the
  // rounding never depends on when a copy lands; an odd last page goes alone
  while (k < cw) {
    const uint32_t st = (uint32_t)k % kRL;
    const bool pair = k + 1 < cw;
    const uint32_t st1 = (uint32_t)(k + 1) % kRL;
    if (!mbar_wait_bounded(my_bars + st, ((uint32_t)k / kRL) & 1u, kWaitNs) ||
        (pair && !mbar_wait_bounded(my_bars + st1, ((uint32_t)(k + 1) / kRL) & 1u, kWaitNs))) {
      if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
      dead = true;
      break;
    }
    const int lp = geom_page(ge, v_lo + warp + k * kWL);
    const bool ok = (vbits >> st) & 1u;
    const int j0 = lp * kPageTok + r;
    if (pair) {
      const int lp1 = geom_page(ge, v_lo + warp + (k + 1) * kWL);
      const bool ok1 = (vbits >> st1) & 1u;
      const int j1 = lp1 * kPageTok + r;
      pages_compute<F>(A, qf, my_stages + st * kStg, ok && geom_has(ge, j0),
                       ok && geom_has(ge, j0 + 8), my_stages + st1 * kStg,
                       ok1 && geom_has(ge, j1), ok1 && geom_has(ge, j1 + 8), true, p.scale_log2,
                       lane);
      __syncwarp();
      if (k + kRL < cw) issue(k + kRL);
      if (k + 1 + kRL < cw) issue(k + 1 + kRL);
      k += 2;
    } else {
      pages_compute<F>(A, qf, my_stages + st * kStg, ok && geom_has(ge, j0),
                       ok && geom_has(ge, j0 + 8), nullptr, false, false, false, p.scale_log2,
                       lane);
      __syncwarp();
      if (k + kRL < cw) issue(k + kRL);
      k += 1;
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int n = warp + i * kWL;
    if (n < g) {
      const float acc = bf16_lo_to_f32(sq[i][0]) * bf16_lo_to_f32(sk0) +
                        bf16_hi_to_f32(sq[i][0]) * bf16_hi_to_f32(sk0) +
                        bf16_lo_to_f32(sq[i][1]) * bf16_lo_to_f32(sk1) +
                        bf16_hi_to_f32(sq[i][1]) * bf16_hi_to_f32(sk1);
      const float sn = warp_sum(acc) * p.scale_log2;
      if (lane == 0) s_snew[n] = sn;
    }
  }
  // a warp that gave up on a barrier first waits (bounded) for the copies it still has in
  // flight; then every warp is done with the stages, which become the merge area
  if (dead) {
    for (int kk = k; kk < cw && kk < k + kRL; ++kk)
      (void)mbar_wait_bounded(my_bars + (kk % kRL), ((uint32_t)kk / kRL) & 1u, kWaitNs);
  }
  __syncthreads();
  warp_flush(A, merge_o + warp * g * kMergeStride, merge_ml + warp * 16, g, lane);
  __syncthreads();
  cluster_wait();
  // this CTA's merged partial, into slot `rank` of rank 0's inbox (plain stores through the
  // cluster window for rank != 0)
  float* dst_o = rank == 0 ? inbox_o : cluster.map_shared_rank(inbox_o, 0);
  float* dst_ml = rank == 0 ? inbox_ml : cluster.map_shared_rank(inbox_ml, 0);
  for (int idx = tid; idx < g * 128; idx += kThreadsL) {
    const int n = idx >> 7, d = idx & 127;
    float M, L, O;
    cta_merge<kWL>(merge_o, merge_ml, g, n, d, M, L, O);
    dst_o[((size_t)rank * g + n) * 128 + d] = O;
    if (d == 0) {
      dst_ml[((size_t)rank * g + n) * 2] = M;
      dst_ml[((size_t)rank * g + n) * 2 + 1] = L;
    }
  }
  __syncthreads();
  if (rank != 0) {
    // the barrier above orders every thread's inbox writes before this release
    if (tid == 0) mbar_arrive_remote(mapa_shared(smem_u32(&inbox_bar), 0));
    return;
  }
  if (C > 1) {
    // bounded: every other rank arrives after its own bounded page waits
    bool ok = mbar_try_wait_cluster(&inbox_bar, 0u);
    if (!ok) {
      const uint64_t t0 = global_timer_ns();
      while (!(ok = mbar_try_wait_cluster(&inbox_bar, 0u)))
        if (global_timer_ns() - t0 > 5 * kWaitNs) break;
      if (!ok && tid == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
    }
  }
  if (ge.active) {
    // the cluster's partials plus the staged token, in rank order: g*128 outputs
    const int n_out = g * 128;
#pragma unroll
    for (int i = 0; i < (8 * 128) / kThreadsL; ++i) {
      const int idx = tid + i * kThreadsL;
      if (idx >= n_out) break;
      const int n = idx >> 7, d = idx & 127;
      const float snew = s_snew[n];
      float Mr[kMaxCluster], Lr[kMaxCluster], Or[kMaxCluster];
      float M = snew;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        if (q < C) {
          Mr[q] = inbox_ml[((size_t)q * g + n) * 2];
          Lr[q] = inbox_ml[((size_t)q * g + n) * 2 + 1];
          Or[q] = inbox_o[((size_t)q * g + n) * 128 + d];
          M = fmaxf(M, Mr[q]);
        }
      }
      const float wn = exp2f(snew - M);
      const float vd = v_staged[i];
      float L = wn, O = wn * vd;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        if (q < C && Mr[q] != -INFINITY) {
          const float w = exp2f(Mr[q] - M);
          L += w * Lr[q];
          O += w * Or[q];
        }
      }
      p.out[((size_t)b * p.Hq + h * g + n) * 128 + d] = O / L;
    }
  }
}

// ------------------------------------------------------------ full set: persistent grid
template <int F>
__global__ void __launch_bounds__(kThreads, Fmt<F>::kMinCtas)
attn_full_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const AttnParams p) {
  constexpr int kR = Fmt<F>::kR;
  constexpr int kStg = Fmt<F>::kStage;
  constexpr int kQueueLow = kR + kChunk;   // queue length that triggers the next claim
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + (Fmt<F>::kAlign - 1)) & ~uintptr_t(Fmt<F>::kAlign - 1));
  const int g = p.g;
  float* merge_o = reinterpret_cast<float*>(stages + kW * kR * kStg);   // [W][g][132]
  float* merge_ml = merge_o + kW * g * kMergeStride;                  // [W][8][2]
  float* cpart_o = merge_ml + kW * 16;                                // combine scratch
  __shared__ __align__(8) uint64_t bars[kW * kR];
  __shared__ int s_t[ODA_MAX_BATCH];
  __shared__ int s_nv[ODA_MAX_BATCH];
  __shared__ int s_us[ODA_MAX_BATCH + 1];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, Hkv = p.Hkv;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kW * kR; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    if (F == 0) {
      prefetch_tensormap(&tmA);
      if (!p.kv_single) prefetch_tensormap(&tmB);
    }
  }
  // ---- per-sequence geometry and unit prefix sums (identical in every CTA)
  for (int b = tid; b < B; b += kThreads) {
    const int t = __ldcg(p.pos + b);
    const bool wanted = __ldcg(p.flag + b) != 0;
    const Geom ge = make_geom(t, 1, p.sinks, p.window, p.max_pages, wanted);
    s_t[b] = t;
    s_nv[b] = ge.active ? max(1, geom_pages(ge)) : 0;
    if (wanted && !ge.active && blockIdx.x == 0) atomicOr(p.err, ODA_DEVERR_POS_RANGE);
  }
  __syncthreads();
  if (warp == 0) {
    int running = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      const int cnt = (b < B) ? Hkv * s_nv[b] : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b < B) s_us[b] = running + incl - cnt;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_us[B] = running;
  }
  __syncthreads();
  // G = min(grid, U) CTAs share the units, so that every one of them owns at least one unit
  // and the CTAs covering a (b, h) are exactly the consecutive range found by cta_of.
  const long long U = s_us[B];
  const long long G = U < (long long)gridDim.x ? U : (long long)gridDim.x;
  int u0 = 0, u1 = 0;
  // Ranges go to CTAs through the stride permutation v = c * perm mod grid (perm coprime to
  // the grid): the CTAs covering one (b, h) are then spread over the dispatch order instead of
  // being dispatched together, so no (b, h) is left to the CTAs that start last.
  const int vc = (int)(((long long)blockIdx.x * p.cta_perm) % gridDim.x);
  if ((long long)vc < G) {
    u0 = (int)(vc * U / G);
    u1 = (int)((vc + 1) * U / G);
  }
  uint8_t* my_stages = stages + warp * kR * kStg;
  uint64_t* my_bars = bars + warp * kR;

  // ---- this warp's copy stream.  The pages of a (b, h) are split into chunks of kChunk
  // pages.  Every warp of a CTA whose range starts in (b, h) owns one fixed chunk (rank-major,
  // so it can be fetched before the dependency wait); the remaining chunks are claimed from the
  // (b, h)'s counter by the warps of all CTAs covering it, so that CTAs on faster SMs take more
  // of them.  A CTA whose first (b, h) began before its range and that has more (b, h) after it
  // claims there no more than its own share: the CTAs for which that (b, h) is the last one
  // claim the rest, so a CTA covering several short (b, h) does not fall behind on the ones
  // only it covers.  Claimed pages wait in a per-warp queue held one entry per lane (entry i in
  // lane i % 32); copies run kR pages ahead of the arithmetic and may cross into the next segment.
  uint32_t issued = 0, consumed = 0, vbits = 0;
  uint32_t f_head = 0, f_tail = 0;            // queue entries [f_head, f_tail)
  int f_phys = -1, f_h = 0, f_lp = 0, f_seg = 0;
  int st_lp = 0, st_seg = 0;                  // lane st: logical page and segment of stage st
  bool dead = false;
  // claim side (warp-uniform; `pend` lives in lane 0)
  int is_seg = 0, is_u = u0, is_b = 0, is_h = 0, is_bh = 0, is_nv = 0, is_ncache = 0;
  int is_nch = 0, is_base = 0, is_fixed = -1, pend = 0;
  int is_rank = 0, is_nc = 1, is_next = 0;   // fixed pattern: rank among covering CTAs, count, cursor
  int is_cap = 0x7fffffff, is_taken = 0;      // this warp's claim limit in the segment, claims taken
  bool is_done = u0 >= u1, claims_ok = false, has_pend = false;
  auto enter_seg = [&](bool first) {
    const Seg cs_ = decode_seg(is_u, u1, s_us, s_nv, B, Hkv);
    is_b = cs_.b;
    is_h = cs_.h;
    is_bh = cs_.b * Hkv + cs_.h;
    is_nv = cs_.nv;
    is_ncache = s_t[cs_.b] - 1;
    is_nch = (is_nv + kChunk - 1) / kChunk;
    // CTAs whose range starts inside this (b, h): [cfs, cfe); their warps own chunks
    // 0 .. (cfe - cfs) * kW - 1, one each; claims hand out the chunks after those
    const long long s0 = cs_.s0, s1 = (long long)cs_.s0 + cs_.nv;
    const long long cfs = (s0 * G + U - 1) / U;
    const long long cfe = min(G, (s1 * G + U - 1) / U);
    is_base = (int)(cfe - cfs) * kW;
    is_fixed = first ? (int)((long long)vc - cfs) * kW + warp : -1;
    has_pend = false;
    is_taken = 0;
    is_cap = 0x7fffffff;
    if (first && s0 < u0 && s1 < u1) {
      // the CTA's share [u0, s1) in chunks, less the warps' fixed chunks, split over the warps
      const int share = (int)((s1 - u0 + kChunk - 1) / kChunk);
      is_cap = max(0, (share - kW + kW - 1) / kW);
    }
    if (p.deterministic) {
      // fixed pattern: chunk j goes to covering CTA j % nc, and within it to warp (j / nc) % kW
      const int c0 = cta_of(cs_.s0, U, G), c1 = cta_of(s1 - 1, U, G);
      is_nc = c1 - c0 + 1;
      is_rank = vc - c0;
      is_next = 0;
      is_fixed = -1;
      return;
    }
    if (claims_ok && is_taken < is_cap) {
      if (lane == 0) pend = atomicAdd(p.claims + is_bh, 1);
      has_pend = true;
      ++is_taken;
    }
  };
  // lanes look up the physical pages of chunk c of the claim segment into queue entries
  auto push_chunk = [&](int c) {
    const int first = c * kChunk;
    const int np = min(kChunk, is_nv - first);
    const int j = (int)(((uint32_t)lane - f_tail) & 31u);
    if (j < np) {
      const int lp = first + j;
      int phys = -1;   // an empty cache keeps one unit that loads nothing
      if (is_ncache > 0) {
        const int e = __ldcg(p.page_table + (size_t)is_b * p.max_pages + lp);
        phys = (e >= 0 && (int64_t)e < p.n_pool_pages) ? e : -2;
        if (phys == -2) atomicOr(p.err, ODA_DEVERR_PAGE_RANGE);
      }
      f_phys = phys;
      f_h = is_h;
      f_lp = lp;
      f_seg = is_seg;
    }
    f_tail += (uint32_t)np;
  };
  auto next_segment = [&]() {
    is_u += decode_seg(is_u, u1, s_us, s_nv, B, Hkv).n;
    ++is_seg;
    if (is_u >= u1) is_done = true;
    else enter_seg(false);
  };
  // queue one more chunk, or move the claim side to the next segment
  auto top_up = [&]() {
    if (is_done || dead || f_tail - f_head >= (uint32_t)kQueueLow) return;
    if (p.deterministic) {   // this warp's i-th chunk is rank + nc * (warp + kW * i)
      const int c = is_rank + is_nc * (warp + kW * is_next);
      if (c < is_nch) {
        ++is_next;
        push_chunk(c);
      } else {
        next_segment();
      }
      return;
    }
    if (is_fixed >= 0) {
      const int c = is_fixed;
      is_fixed = -1;
      if (c < is_nch) {
        push_chunk(c);
        return;
      }
    }
    if (!claims_ok) return;
    if (!has_pend) {
      if (is_taken >= is_cap) {   // this warp's share of the segment is taken
        next_segment();
        return;
      }
      if (lane == 0) pend = atomicAdd(p.claims + is_bh, 1);
      has_pend = true;
      ++is_taken;
    }
    const int c = is_base + __shfl_sync(0xffffffffu, pend, 0);
    has_pend = false;
    if (c < is_nch) {
      push_chunk(c);
      // the next claim is taken ahead (it is always used: a claim is never dropped)
      if (is_taken < is_cap) {
        if (lane == 0) pend = atomicAdd(p.claims + is_bh, 1);
        has_pend = true;
        ++is_taken;
      }
    } else {
      next_segment();
    }
  };
  // copy the queue head into the next stage
  auto issue_one = [&]() {
    const int src = (int)(f_head & 31u);
    const int phys = __shfl_sync(0xffffffffu, f_phys, src);
    const int hh = __shfl_sync(0xffffffffu, f_h, src);
    const int lp = __shfl_sync(0xffffffffu, f_lp, src);
    const int sg = __shfl_sync(0xffffffffu, f_seg, src);
    const uint32_t st = issued % kR;
    if (lane == src) {
      if (phys >= 0)
        issue_any<F>(my_stages + st * kStg, my_bars + st, &tmA, &tmB, p, phys, hh);
      else
        mbar_arrive(my_bars + st);
    }
    if (lane == (int)st) {
      st_lp = lp;
      st_seg = sg;
    }
    vbits = phys >= 0 ? (vbits | (1u << st)) : (vbits & ~(1u << st));
    ++issued;
    ++f_head;
  };
  // keep kR copies in flight while pages remain
  auto pump = [&]() {
    while (!dead && issued - consumed < (uint32_t)kR) {
      if (f_head == f_tail) {
        top_up();
        if (f_head == f_tail) {
          if (is_done || (!claims_ok && !p.deterministic)) break;
          continue;
        }
      }
      issue_one();
    }
  };
  if (!is_done) enter_seg(true);
  pump();
  // Everything above reads only the cache, the page table and positions/flags, which an
  // attention launch never writes; the previous launch of the stream may still be running
  // (programmatic dependent launch).  Wait for it before claiming, reading q or writing.
  grid_dependency_wait();
  grid_dependents_launch();
  claims_ok = true;
  if (!is_done && is_fixed < 0 && !p.deterministic && is_taken < is_cap) {
    if (lane == 0) pend = atomicAdd(p.claims + is_bh, 1);
    has_pend = true;
    ++is_taken;
  }

  // ---- segments of this CTA, in order
  int cseg = 0;
  for (int seg_u = u0; seg_u < u1; ++cseg) {
    const Seg cs = decode_seg(seg_u, u1, s_us, s_nv, B, Hkv);
    const int b = cs.b, h = cs.h;
    const int n_cache = s_t[b] - 1;
    QFrag<F> qf;
    load_q<F>(qf, p, b, h, lane);
    WarpAcc A;
    acc_init(A);
    const int r = lane >> 2;
    while (!dead) {
      if (consumed == issued) {
        pump();
        if (consumed == issued) break;
      }
      const uint32_t st = consumed % kR;
      if (__shfl_sync(0xffffffffu, st_seg, (int)st) != cseg) break;  // a later segment's page
      if (!mbar_wait_bounded(my_bars + st, (consumed / kR) & 1u, kWaitNs)) {
        if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
        dead = true;
        break;
      }
      const bool ok = (vbits >> st) & 1u;
      const int lp = __shfl_sync(0xffffffffu, st_lp, (int)st);
      const int j0 = lp * kPageTok + r;
      // An even page and the next page of its chunk go through one softmax step.  Chunks are
      // queued whole and copies run kR >= 2 ahead, so the partner is always issued by now: the
      // pairing depends only on page numbers, never on copy timing.
      bool pair = false;
      const uint32_t st1 = (consumed + 1) % kR;
      if ((lp & 1) == 0 && consumed + 1 < issued)
        pair = __shfl_sync(0xffffffffu, st_seg, (int)st1) == cseg &&
               __shfl_sync(0xffffffffu, st_lp, (int)st1) == lp + 1;
      if (pair) {
        if (!mbar_wait_bounded(my_bars + st1, ((consumed + 1) / kR) & 1u, kWaitNs)) {
          if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
          dead = true;
          break;
        }
        const bool ok1 = (vbits >> st1) & 1u;
        const int j1 = j0 + kPageTok;
        pages_compute<F>(A, qf, my_stages + st * kStg, ok && j0 < n_cache, ok && j0 + 8 < n_cache,
                         my_stages + st1 * kStg, ok1 && j1 < n_cache, ok1 && j1 + 8 < n_cache, true,
                         p.scale_log2, lane);
        consumed += 2;
      } else {
        pages_compute<F>(A, qf, my_stages + st * kStg, ok && j0 < n_cache, ok && j0 + 8 < n_cache,
                         nullptr, false, false, false, p.scale_log2, lane);
        ++consumed;
      }
      __syncwarp();
      top_up();
      pump();
    }
    warp_flush(A, merge_o + warp * g * kMergeStride, merge_ml + warp * 16, g, lane);
    __syncthreads();
    // ---- merge the warps into this segment's partial (one per query head of the group)
    const int bh = b * Hkv + h;
    const int slot = vc + bh;
    for (int idx = tid; idx < g * 128; idx += kThreads) {
      const int n = idx >> 7, d = idx & 127;
      float M, L, O;
      cta_merge<kW>(merge_o, merge_ml, g, n, d, M, L, O);
      p.part_o[((size_t)slot * g + n) * 128 + d] = O;
      if (d == 0) {
        p.part_ml[((size_t)slot * g + n) * 2] = M;
        p.part_ml[((size_t)slot * g + n) * 2 + 1] = L;
      }
    }
    // publish: the CTA barrier orders every thread's partial writes before thread 0's
    // gpu-scope fence and count; the CTA that completes the count reads all partials
    __syncthreads();
    const int c_first = cta_of(cs.s0, U, G), c_last = cta_of(cs.s0 + cs.nv - 1, U, G);
    const int nparts = c_last - c_first + 1;
    if (tid == 0) {
      __threadfence();
      s_last = (atomicAdd(&p.counters[bh], 1) == nparts - 1);
      if (s_last) __threadfence();
    }
    __syncthreads();
    if (s_last) {
      // ---- last CTA of (b, h): merge the nparts partials and the staged current token in one
      // online pass.  Each round loads kMergeRows partial rows of a head together with their
      // (m, l) and folds them into a running (M, L, O), so nparts = 37 costs two L2 round trips.
      const int slot0 = c_first + bh;
      const size_t rs = (size_t)g * 32;   // float4 stride between partial rows
      // (M, L, O) of head n over the partials s = sub, sub + step, ... (lane l: dims 4l..4l+3)
      auto fold = [&](int n, int sub, int step, float& M, float& L, float4& acc) {
        const float4* base =
            reinterpret_cast<const float4*>(p.part_o + ((size_t)slot0 * g + n) * 128) + lane;
        const float* mlb = p.part_ml + ((size_t)slot0 * g + n) * 2;
        M = -INFINITY;
        L = 0.f;
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = sub; s0 < nparts; s0 += kMergeRows * step) {
          float4 v[kMergeRows];
          const int sj = s0 + lane * step;   // lane j < kMergeRows holds (m, l) of row j
          float mj = -INFINITY, lj = 0.f;
          if (lane < kMergeRows && sj < nparts) {
            mj = __ldcg(mlb + (size_t)sj * g * 2);
            lj = __ldcg(mlb + (size_t)sj * g * 2 + 1);
          }
#pragma unroll
          for (int j = 0; j < kMergeRows; ++j) {
            const int sr = s0 + j * step;
            v[j] = sr < nparts ? __ldcg(base + (size_t)sr * rs) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          float mb = mj;
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o2));
          const float Mn = fmaxf(M, mb);
          if (Mn == -INFINITY) continue;   // no tokens so far (empty partials)
          const float sc = (M == -INFINITY) ? 0.f : exp2f(M - Mn);
          const float wj = (mj == -INFINITY) ? 0.f : exp2f(mj - Mn);
          acc.x *= sc;
          acc.y *= sc;
          acc.z *= sc;
          acc.w *= sc;
          L = L * sc + warp_sum(wj * lj);
#pragma unroll
          for (int j = 0; j < kMergeRows; ++j) {
            const float w = __shfl_sync(0xffffffffu, wj, j);
            acc.x += w * v[j].x;
            acc.y += w * v[j].y;
            acc.z += w * v[j].z;
            acc.w += w * v[j].w;
          }
          M = Mn;
        }
      };
      // the staged current token of head n: its words are loaded before the partial rounds
      struct Staged { uint32_t qa0, qa1, ka0, ka1, v01, v23; };
      auto staged_words = [&](int n) {
        const uint32_t* qrow = p.q + ((size_t)b * p.Hq + h * g + n) * 64;
        const uint32_t* krow = p.k_new + ((size_t)b * p.Hkv + h) * 64;
        const uint32_t* vp = p.v_new + ((size_t)b * p.Hkv + h) * 64 + 2 * lane;
        return Staged{qrow[lane], qrow[lane + 32], krow[lane], krow[lane + 32], vp[0], vp[1]};
      };
      // adds the staged current token of head n and writes the output row
      auto finish = [&](int n, const Staged& sw, float M, float L, float4 acc) {
        const uint32_t qa0 = sw.qa0, qa1 = sw.qa1, ka0 = sw.ka0, ka1 = sw.ka1;
        const uint32_t v01 = sw.v01, v23 = sw.v23;
        const float snew = warp_sum(bf16_lo_to_f32(qa0) * bf16_lo_to_f32(ka0) +
                                    bf16_hi_to_f32(qa0) * bf16_hi_to_f32(ka0) +
                                    bf16_lo_to_f32(qa1) * bf16_lo_to_f32(ka1) +
                                    bf16_hi_to_f32(qa1) * bf16_hi_to_f32(ka1)) * p.scale_log2;
        const float Mf = fmaxf(M, snew);
        const float wa = (M == -INFINITY) ? 0.f : exp2f(M - Mf), wn = exp2f(snew - Mf);
        const float inv = 1.0f / (L * wa + wn);
        float4 o;
        o.x = (acc.x * wa + wn * bf16_lo_to_f32(v01)) * inv;
        o.y = (acc.y * wa + wn * bf16_hi_to_f32(v01)) * inv;
        o.z = (acc.z * wa + wn * bf16_lo_to_f32(v23)) * inv;
        o.w = (acc.w * wa + wn * bf16_hi_to_f32(v23)) * inv;
        reinterpret_cast<float4*>(p.out + ((size_t)b * p.Hq + h * g + n) * 128)[lane] = o;
      };
      if (g >= kW) {
        // a warp per head: heads warp, warp + kW, ...
        for (int n = warp; n < g; n += kW) {
          const Staged sw = staged_words(n);
          float M, L;
          float4 acc;
          fold(n, 0, 1, M, L, acc);
          finish(n, sw, M, L, acc);
        }
      } else {
        // kW / g warps share a head's partials, then warp n (< g) combines them
        // (g = 3: warps 0..2 take one head each, warp 3 idles)
        const int wph = kW / g, n = warp % g, sub = warp / g;
        const Staged sw = staged_words(n);
        float* s_red = cpart_o;   // [kW][132]: O (128), M, L
        float M = -INFINITY, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (sub < wph) fold(n, sub, wph, M, L, acc);
        reinterpret_cast<float4*>(s_red + warp * 132)[lane] = acc;
        if (lane == 0) {
          s_red[warp * 132 + 128] = M;
          s_red[warp * 132 + 129] = L;
        }
        __syncthreads();
        if (warp < g) {
          float Mt = -INFINITY;
          for (int k2 = 0; k2 < wph; ++k2) Mt = fmaxf(Mt, s_red[(k2 * g + warp) * 132 + 128]);
          float Lt = 0.f;
          float4 at = make_float4(0.f, 0.f, 0.f, 0.f);
          if (Mt != -INFINITY) {
            for (int k2 = 0; k2 < wph; ++k2) {
              const float* r = s_red + (k2 * g + warp) * 132;
              const float mk = r[128];
              if (mk == -INFINITY) continue;
              const float w = exp2f(mk - Mt);
              const float4 rv = reinterpret_cast<const float4*>(r)[lane];
              at.x += w * rv.x;
              at.y += w * rv.y;
              at.z += w * rv.z;
              at.w += w * rv.w;
              Lt += w * r[129];
            }
          }
          finish(warp, sw, Mt, Lt, at);
        }
      }
      if (tid == 0) {
        p.counters[bh] = 0;
        p.claims[bh] = 0;
      }
    }
    __syncthreads();
    seg_u += cs.n;
  }
  // a warp that gave up on a barrier waits (bounded) for the copies it still has in flight
  if (dead) {
    for (uint32_t n = consumed; n < issued; ++n)
      (void)mbar_wait_bounded(my_bars + (n % kR), (n / kR) & 1u, kWaitNs);
  }
}

// Index-set enumeration with the kernel's own geometry (tests): one thread per sequence.
__global__ void index_positions_kernel(const int32_t* pos, const int32_t* flag, int B, int mode,
                                       int sinks, int window, int max_pages, int32_t* positions,
                                       int cap, int32_t* counts) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int t = pos[b];
  const bool wanted = (mode == 0) || (flag[b] != 0);
  const Geom ge = make_geom(t, mode, sinks, window, max_pages, wanted);
  if (!ge.active) {
    counts[b] = 0;
    return;
  }
  int32_t* outp = positions + (size_t)b * cap;
  int n = 0;
  const int nv = geom_pages(ge);
  for (int v = 0; v < nv; ++v) {
    const int lp = geom_page(ge, v);
    for (int s = 0; s < kPageTok; ++s) {
      const int j = lp * kPageTok + s;
      if (geom_has(ge, j)) {
        if (n < cap) outp[n] = j + 1;
        ++n;
      }
    }
  }
  if (n < cap) outp[n] = t;
  ++n;
  counts[b] = min(n, cap);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                              CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  }
  return fn;
}

// Tensor maps of one layer's pools [n_pages][Hkv][16][128] bf16, seen as rows of 128 values
// split into two 64-value (128-byte) halves: dims {64, rows, 2} with byte strides {256, 128},
// box {64, 16, 2}, 128-byte swizzle, so a box lands in shared memory as [half][row][64].
// When V lies above K a fourth dimension of stride v - k selects the pool, and one
// {64, 16, 2, 2} box brings K and V of a page together.
oda_status encode_kv(CUtensorMap* a, CUtensorMap* b, int* single, const void* k, const void* v,
                     int64_t n_pages, int Hkv) {
  EncodeFn enc = get_encode();
  if (!enc) return set_error(ODA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t rows = (cuuint64_t)n_pages * Hkv * kPageTok;
  const uintptr_t ka = reinterpret_cast<uintptr_t>(k), va = reinterpret_cast<uintptr_t>(v);
  const uint64_t kv_stride = va > ka ? (uint64_t)(va - ka) : 0;
  cuuint32_t box[4] = {64, kPageTok, 2, 2};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  if (kv_stride > 0 && kv_stride % 16 == 0 && kv_stride < (uint64_t(1) << 40)) {
    cuuint64_t dims[4] = {64, rows, 2, 2};
    cuuint64_t strides[3] = {256, 128, kv_stride};
    CUresult r = enc(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(k), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r == CUDA_SUCCESS) {
      *b = *a;
      *single = 1;
      return ODA_OK;
    }
  }
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {256, 128};
  const void* base[2] = {k, v};
  CUtensorMap* m[2] = {a, b};
  for (int i = 0; i < 2; ++i) {
    CUresult r = enc(m[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base[i]), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
      return set_error(ODA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  }
  *single = 0;
  return ODA_OK;
}

}  // namespace

// Stride of the full-set CTA -> range permutation: near a quarter of the grid, coprime to it.
int cta_stride(int grid) {
  if (grid <= 2) return 1;
  for (int k = grid / 4 + 1; k < grid; ++k) {
    int a = k, b = grid;
    while (b) {
      const int t = a % b;
      a = b;
      b = t;
    }
    if (a == 1) return k;
  }
  return 1;
}

// stages | merge_o [W][g][132] | merge_ml [W][16] | CTA partial / combine scratch
template <int F>
int full_smem_bytes(int g) {
  const int tail = g * 130 > kW * 132 ? g * 130 : kW * 132;
  return Fmt<F>::kAlign + kW * Fmt<F>::kR * Fmt<F>::kStage +
         (kW * g * kMergeStride + kW * 16 + tail) * (int)sizeof(float);
}
int attention_smem_bytes(int g) { return full_smem_bytes<0>(g); }
// local set: the merge areas live in the stages (kWL * g * 132 + kWL * 16 + g * 130 floats,
// 38 KB at g = 8, within the ~200 KB of stages)
template <int F>
int local_smem_bytes(int C, int g) {
  return Fmt<F>::kAlign + kWL * Fmt<F>::kRL * Fmt<F>::kStage + C * g * 130 * (int)sizeof(float);
}

// Dynamic shared memory the local kernels may use (the device's opt-in limit less their static
// shared memory), set by prepare_attention_kernel; it bounds the cluster size through the inbox.
int g_local_dyn_max[2] = {0, 0};

// Sets the shared-memory limits of both kernels in both page formats and returns the
// persistent full-set grid size for group size g per format (ctas[0] bf16, ctas[1] fp8).  The
// limit is a per-function setting shared by every context of the process, so it is always set
// to the largest group's need (g = 8): a context created later with a smaller g must not lower
// it under a launch of an earlier context.
oda_status prepare_attention_kernel(int g, int n_sms, int* ctas) {
  oda_status st = check_cuda(
      cudaFuncSetAttribute(attn_full_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           full_smem_bytes<0>(8)),
      "cudaFuncSetAttribute(full attention)");
  if (st == ODA_OK)
    st = check_cuda(cudaFuncSetAttribute(attn_full_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         full_smem_bytes<1>(8)),
                    "cudaFuncSetAttribute(full attention, fp8)");
  int dev = 0, optin = 0;
  if (st == ODA_OK) st = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (st == ODA_OK)
    st = check_cuda(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev),
                    "cudaDeviceGetAttribute");
  const void* local_k[2] = {reinterpret_cast<const void*>(attn_local_kernel<0>),
                            reinterpret_cast<const void*>(attn_local_kernel<1>)};
  for (int f = 0; f < 2 && st == ODA_OK; ++f) {
    cudaFuncAttributes fa;
    st = check_cuda(cudaFuncGetAttributes(&fa, local_k[f]), "cudaFuncGetAttributes(local attention)");
    if (st != ODA_OK) break;
    g_local_dyn_max[f] = optin - (int)fa.sharedSizeBytes;
    const int base = f == 0 ? local_smem_bytes<0>(1, 1) : local_smem_bytes<1>(1, 1);
    if (g_local_dyn_max[f] < base) return set_error(ODA_ERR_UNSUPPORTED, "local attention: shared memory too small");
    st = check_cuda(cudaFuncSetAttribute(local_k[f], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         g_local_dyn_max[f]),
                    "cudaFuncSetAttribute(local attention)");
  }
  if (st != ODA_OK) return st;
  for (int f = 0; f < 2; ++f) {
    int occ = 0;
    st = f == 0 ? check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, attn_full_kernel<0>,
                                                                          kThreads, full_smem_bytes<0>(g)),
                             "cudaOccupancyMaxActiveBlocksPerMultiprocessor")
                : check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, attn_full_kernel<1>,
                                                                          kThreads, full_smem_bytes<1>(g)),
                             "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (st != ODA_OK) return st;
    occ = std::max(1, std::min(occ, f == 0 ? Fmt<0>::kMinCtas : Fmt<1>::kMinCtas));
    ctas[f] = n_sms * occ;
    // the combine keeps one weight per partial and head in the merge area
    if (ctas[f] > kW * kMergeStride) return set_error(ODA_ERR_UNSUPPORTED, "too many CTAs for the merge area");
  }
  return ODA_OK;
}

oda_status launch_attention(oda_ctx* ctx, const KvPool& pool, const int32_t* page_table,
                            const int32_t* pos, const int32_t* flag, const void* q,
                            const void* k_new, const void* v_new, float* out, int mode,
                            cudaStream_t stream) {
  const oda_config& cf = ctx->cfg;
  const int F = pool.fmt;
  if (!pool.k || (F == 0 && !pool.v) || !page_table || !pos || !q || !k_new || !v_new || !out ||
      (mode == 1 && !flag))
    return set_error(ODA_ERR_INVALID_ARG, "attention: null pointer argument");
  if (pool.n_pages <= 0 || pool.n_pages * (int64_t)cf.n_kv_heads * kPageTok > INT32_MAX)
    return set_error(ODA_ERR_INVALID_ARG, "attention: n_pages out of range (%lld)",
                     (long long)pool.n_pages);
  if ((reinterpret_cast<uintptr_t>(pool.k) | reinterpret_cast<uintptr_t>(pool.v)) & 15)
    return set_error(ODA_ERR_INVALID_ARG, "attention: K/V pools must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_new) |
       reinterpret_cast<uintptr_t>(v_new) | reinterpret_cast<uintptr_t>(out)) & 3)
    return set_error(ODA_ERR_INVALID_ARG, "attention: q/k_new/v_new/out must be 4-byte aligned");
  CUtensorMap tmA, tmB;
  memset(&tmA, 0, sizeof tmA);
  memset(&tmB, 0, sizeof tmB);
  int kv_single = 0;
  oda_status st = ODA_OK;
  if (F == 0) {
    st = encode_kv(&tmA, &tmB, &kv_single, pool.k, pool.v, pool.n_pages, cf.n_kv_heads);
    if (st != ODA_OK) return st;
  }
  AttnParams p;
  p.kv_single = kv_single;
  p.cta_perm = 1;
  p.deterministic = cf.deterministic;
  p.page_table = page_table;
  p.pos = pos;
  p.flag = flag;
  p.kv8 = F == 1 ? static_cast<const uint8_t*>(pool.k) : nullptr;
  p.q = static_cast<const uint32_t*>(q);
  p.k_new = static_cast<const uint32_t*>(k_new);
  p.v_new = static_cast<const uint32_t*>(v_new);
  p.out = out;
  p.part_o = ctx->part_o;
  p.part_ml = ctx->part_ml;
  p.counters = ctx->attn_cnt;
  p.claims = ctx->attn_cnt + (size_t)cf.batch * cf.n_kv_heads;
  p.err = ctx->err;
  p.n_pool_pages = pool.n_pages;
  p.B = cf.batch;
  p.Hq = cf.n_q_heads;
  p.Hkv = cf.n_kv_heads;
  p.g = ctx->g;
  p.max_pages = cf.max_pages;
  p.sinks = cf.sinks;
  p.window = cf.window;
  p.mode = mode;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  // cluster size of the local kernel: about one CTA per SM (each CTA's page rings take most of
  // an SM's shared memory), at most 8 per (b, h)
  const int pairs = cf.batch * cf.n_kv_heads;
  p.cluster = std::max(1, std::min(kMaxCluster, ctx->n_sms / pairs));
  // rank 0's inbox holds every rank's partial: a smaller cluster where it would not fit
  while (p.cluster > 1 && (F == 0 ? local_smem_bytes<0>(p.cluster, ctx->g) : local_smem_bytes<1>(p.cluster, ctx->g)) >
                              g_local_dyn_max[F])
    --p.cluster;

  // Consecutive attention launches of one context overlap when the context allows it: the
  // later one may start (and prefetch its pages) while the earlier one finishes; it waits
  // before reading q or writing.
  cudaLaunchConfig_t lc = {};
  lc.blockDim = dim3(mode == 0 ? kThreadsL : kThreads);
  lc.dynamicSmemBytes = mode == 0 ? (F == 0 ? local_smem_bytes<0>(p.cluster, ctx->g)
                                              : local_smem_bytes<1>(p.cluster, ctx->g))
                                  : (F == 0 ? full_smem_bytes<0>(ctx->g) : full_smem_bytes<1>(ctx->g));
  lc.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (cf.overlap_layers && ctx->prev_attention) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (mode == 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    lc.gridDim = dim3(pairs * p.cluster);
  } else {
    lc.gridDim = dim3(ctx->attn_ctas[F]);
    p.cta_perm = cta_stride(ctx->attn_ctas[F]);
  }
  lc.attrs = attr;
  lc.numAttrs = na;
  if (mode == 0)
    st = F == 0 ? check_cuda(cudaLaunchKernelEx(&lc, attn_local_kernel<0>, tmA, tmB, p), "local attention launch")
                : check_cuda(cudaLaunchKernelEx(&lc, attn_local_kernel<1>, tmA, tmB, p), "local attention launch");
  else
    st = F == 0 ? check_cuda(cudaLaunchKernelEx(&lc, attn_full_kernel<0>, tmA, tmB, p), "full attention launch")
                : check_cuda(cudaLaunchKernelEx(&lc, attn_full_kernel<1>, tmA, tmB, p), "full attention launch");
  ctx->prev_attention = (st == ODA_OK);
  return st;
}

oda_status launch_index_positions(oda_ctx* ctx, int mode, const int32_t* pos, const int32_t* flag,
                                  int32_t* positions, int32_t cap, int32_t* counts,
                                  cudaStream_t stream) {
  if (!pos || !positions || !counts || cap <= 0 || (mode == 1 && !flag) || (mode != 0 && mode != 1))
    return set_error(ODA_ERR_INVALID_ARG, "index_positions: bad argument");
  const oda_config& cf = ctx->cfg;
  ctx->prev_attention = false;
  index_positions_kernel<<<(cf.batch + 31) / 32, 32, 0, stream>>>(
      pos, flag, cf.batch, mode, cf.sinks, cf.window, cf.max_pages, positions, cap, counts);
  return check_cuda(cudaGetLastError(), "index_positions launch");
}


// ------------------------------------------------------------- allocation-free variant
// Callers that must not allocate device memory (a plugin that may only use the buffers its
// host framework hands it, code that runs where a cudaMalloc/cudaFree would synchronise the
// device in a latency-critical loop, or a process whose memory is reserved up front) get
// the full-set attention with its scratch in this file-scope device array instead of a
// context.  Every GPU that loads the library holds the array until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
  unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch on this device
  int n_sms = 0;
  int ctas[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};   // persistent bf16 grid size per group size g
  bool ready = false;
};
constexpr int kNoAllocMaxDevices = 64;
NoAllocDevice g_noalloc[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

// Once per device, with that device current: the array's device address (host code only
// sees a stand-in symbol); once per (device, g): the kernel's shared-memory limit and the
// persistent grid size, from the same occupancy query a context uses, so both entry points
// launch the same grid and split the work the same way.
oda_status noalloc_setup(int g, NoAllocDevice** out, int* ctas) {
  int dev = 0;
  oda_status st = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != ODA_OK) return st;
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return set_error(ODA_ERR_UNSUPPORTED, "noalloc: device %d beyond the supported %d", dev,
                     kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc[dev];
  if (!d.ready) {
    void* ptr = nullptr;
    st = check_cuda(cudaGetSymbolAddress(&ptr, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    if (st != ODA_OK) return st;
    st = check_cuda(cudaDeviceGetAttribute(&d.n_sms, cudaDevAttrMultiProcessorCount, dev),
                    "cudaDeviceGetAttribute");
    if (st != ODA_OK) return st;
    d.scratch = static_cast<unsigned char*>(ptr);
    d.ready = true;
  }
  if (d.ctas[g] == 0) {
    int both[2] = {0, 0};
    st = prepare_attention_kernel(g, d.n_sms, both);
    if (st != ODA_OK) return st;
    d.ctas[g] = both[0];
  }
  *out = &d;
  *ctas = d.ctas[g];
  return ODA_OK;
}

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

oda_status launch_attention_noalloc(const oda_config* cfg, const oda_kv_layer* layer,
                                    const int32_t* page_table, const int32_t* pos,
                                    const int32_t* flag, const void* q, const void* k_new,
                                    const void* v_new, float* out, int32_t* device_error,
                                    cudaStream_t stream) {
  if (!cfg) return set_error(ODA_ERR_INVALID_ARG, "noalloc: cfg is NULL");
  const oda_config& cf = *cfg;
  oda_status st = validate_attention_config(cf, "noalloc");
  if (st != ODA_OK) return st;
  if (!layer || !layer->k || !layer->v || !page_table || !pos || !flag || !q || !k_new || !v_new ||
      !out)
    return set_error(ODA_ERR_INVALID_ARG, "noalloc: null pointer argument");
  if (layer->n_pages <= 0 || layer->n_pages * (int64_t)cf.n_kv_heads * kPageTok > INT32_MAX)
    return set_error(ODA_ERR_INVALID_ARG, "noalloc: n_pages out of range");
  if ((reinterpret_cast<uintptr_t>(layer->k) | reinterpret_cast<uintptr_t>(layer->v)) & 15)
    return set_error(ODA_ERR_INVALID_ARG, "noalloc: K/V pools must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_new) |
       reinterpret_cast<uintptr_t>(v_new) | reinterpret_cast<uintptr_t>(out)) & 3)
    return set_error(ODA_ERR_INVALID_ARG, "noalloc: q/k_new/v_new/out must be 4-byte aligned");
  const int g = cf.n_q_heads / cf.n_kv_heads;
  NoAllocDevice* d = nullptr;
  int ctas = 0;
  st = noalloc_setup(g, &d, &ctas);
  if (st != ODA_OK) return st;
  // scratch layout: completion counters [B*Hkv] | claim counters [B*Hkv] | error word |
  // partial (m, l) | partial O
  const size_t pairs = (size_t)cf.batch * cf.n_kv_heads;
  const size_t slots = (size_t)ctas + pairs;
  const size_t cnt_bytes = ((2 * pairs + 1) * sizeof(int32_t) + 255) / 256 * 256;
  const size_t ml_bytes = (slots * g * 2 * sizeof(float) + 255) / 256 * 256;
  const size_t o_bytes = slots * g * 128 * sizeof(float);
  if (cnt_bytes + ml_bytes + o_bytes > kNoAllocScratchBytes)
    return set_error(ODA_ERR_UNSUPPORTED,
                     "noalloc: needs %zu bytes of scratch for B=%d, Hkv=%d, g=%d; the static "
                     "scratch holds %zu",
                     cnt_bytes + ml_bytes + o_bytes, cf.batch, cf.n_kv_heads, g,
                     kNoAllocScratchBytes);
  int32_t* counters = reinterpret_cast<int32_t*>(d->scratch);
  int32_t* err_word = counters + 2 * pairs;
  float* part_ml = reinterpret_cast<float*>(d->scratch + cnt_bytes);
  float* part_o = reinterpret_cast<float*>(d->scratch + cnt_bytes + ml_bytes);
  // the counters (and the scratch error word) must start at zero on every call
  st = check_cuda(cudaMemsetAsync(counters, 0, (2 * pairs + 1) * sizeof(int32_t), stream),
                  "cudaMemsetAsync(noalloc counters)");
  if (st != ODA_OK) return st;
  CUtensorMap tmA, tmB;
  int kv_single = 0;
  st = encode_kv(&tmA, &tmB, &kv_single, layer->k, layer->v, layer->n_pages, cf.n_kv_heads);
  if (st != ODA_OK) return st;
  AttnParams p;
  p.kv_single = kv_single;
  p.cta_perm = 1;
  p.deterministic = cf.deterministic;
  p.page_table = page_table;
  p.pos = pos;
  p.flag = flag;
  p.q = static_cast<const uint32_t*>(q);
  p.k_new = static_cast<const uint32_t*>(k_new);
  p.v_new = static_cast<const uint32_t*>(v_new);
  p.out = out;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.counters = counters;
  p.claims = counters + pairs;
  p.err = device_error ? device_error : err_word;
  p.n_pool_pages = layer->n_pages;
  p.B = cf.batch;
  p.Hq = cf.n_q_heads;
  p.Hkv = cf.n_kv_heads;
  p.g = g;
  p.max_pages = cf.max_pages;
  p.sinks = cf.sinks;
  p.window = cf.window;
  p.mode = 1;
  p.cluster = 1;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  p.kv8 = nullptr;
  p.cta_perm = cta_stride(ctas);
  attn_full_kernel<0><<<ctas, kThreads, attention_smem_bytes(g), stream>>>(tmA, tmB, p);
  return check_cuda(cudaGetLastError(), "noalloc full attention launch");
}

}  // namespace oda
