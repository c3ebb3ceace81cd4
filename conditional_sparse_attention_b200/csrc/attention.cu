// Split-KV flash-decode over a paged bf16 KV cache for the two ODA index sets.
//
// Method: "On-Demand Attention：让语言模型按需读取完整历史" (method notes) §2.1, eq. o_t and
// eq. S^F / S^L: one decode query per sequence attends, per layer, over either the local set
// S^L_t = {1..min(s,t)} U {max(1,t-w+1)..t} or the full set S^F_t = {1..t} of one retained
// cache; the current token's K,V (position t) come from the branch's staging, not the cache.
//
// Kernel design (sm_100a):
//   * persistent grid (2 CTAs per SM); a work item is (sequence b, KV head h, split of
//     pages); items are enumerated on the device from pos[] (and flag[] for the full set),
//     so the full retry of unflagged sequences costs nothing and the host never syncs;
//   * each of the 4 warps of a CTA streams every 4th page of its item through a private
//     3-stage ring: one 2-D TMA tile load per 64-dim half of K and V (4 x 2 KiB per page,
//     128-byte swizzle), completion on an mbarrier (bounded waits, no spin without limit);
//   * scores S = K Q^T with tokens as the M dimension and the g query heads of the GQA group
//     as N (mma.sync m16n8k16 bf16 -> fp32); online softmax in the exp2 domain with
//     warp-shuffle column maxima; P^T reaches the PV product through movmatrix.trans; P is
//     split into bf16 hi + lo parts so the PV product keeps ~fp32 accuracy;
//   * per item, the 4 warp states are merged in shared memory into one (m, l, acc[128])
//     partial per query head; the last CTA to finish a (b, h) (completion counter, no
//     spin-wait) merges all splits plus the staged current token and writes o.
#include <cmath>
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace oda {
namespace {

constexpr int kW = 4;                 // warps per CTA (each streams its own pages)
constexpr int kR = 3;                 // pages in flight per warp
constexpr int kThreads = kW * 32;
constexpr int kPageTok = 16;
constexpr int kStageBytes = 8192;     // K (4 KiB) + V (4 KiB) of one (page, KV head)
constexpr int kStagesBytes = kW * kR * kStageBytes;
constexpr int kSmemBytes = kStagesBytes + 1024;
constexpr int kMergeStride = 132;     // floats per (warp, head) row of the merge area
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMinSplitPages = 8;
constexpr int kItemsPerCta = 4;       // target work items per CTA when sizing splits
constexpr int kCtasPerSm = 2;

struct AttnParams {
  const int32_t* page_table;
  const int32_t* pos;
  const int32_t* flag;
  const uint32_t* q;      // bf16 pairs [B][Hq][64]
  const uint32_t* k_new;  // bf16 pairs [B][Hkv][64]
  const uint32_t* v_new;
  float* out;             // [B][Hq][128]
  float* part_o;          // [B*Hq][max_splits][128]
  float* part_ml;         // [B*Hq][max_splits][2]
  int32_t* counters;      // [B*Hkv]
  int32_t* err;
  int64_t n_pool_pages;
  int32_t B, Hq, Hkv, g, max_pages, max_splits, sinks, window, mode;
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

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
            const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bars[kW * kR];
  __shared__ int s_t[ODA_MAX_BATCH];
  __shared__ int s_nv[ODA_MAX_BATCH];
  __shared__ int s_start[ODA_MAX_BATCH + 1];
  __shared__ int s_sp;
  __shared__ int s_last;
  __shared__ float s_L[8], s_wnew[8];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, Hkv = p.Hkv, g = p.g;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kW * kR; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  // ---- per-sequence geometry, split size and item prefix sums (identical in every CTA)
  for (int b = tid; b < B; b += kThreads) {
    const int t = p.pos[b];
    const bool wanted = (p.mode == 0) || (p.flag[b] != 0);
    const Geom ge = make_geom(t, p.mode, p.sinks, p.window, p.max_pages, wanted);
    s_t[b] = t;
    s_nv[b] = ge.active ? geom_pages(ge) : -1;
    if (wanted && !ge.active && blockIdx.x == 0) atomicOr(p.err, ODA_DEVERR_POS_RANGE);
  }
  __syncthreads();
  if (warp == 0) {
    long long sum = 0;
    int mx = 0;
    for (int b = lane; b < B; b += 32) {
      const int nv = s_nv[b];
      if (nv > 0) {
        sum += nv;
        mx = max(mx, nv);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const long long target = (long long)kItemsPerCta * gridDim.x;
    int sp = (int)((sum * Hkv + target - 1) / target);
    sp = max(sp, kMinSplitPages);
    sp = max(sp, (mx + p.max_splits - 1) / p.max_splits);
    int running = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      int cnt = 0;
      if (b < B && s_nv[b] >= 0) cnt = Hkv * max(1, (s_nv[b] + sp - 1) / sp);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b < B) s_start[b] = running + incl - cnt;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_start[B] = running;
      s_sp = sp;
    }
  }
  __syncthreads();
  const int total = s_start[B];
  const int SP = s_sp;

  uint32_t issued = 0, consumed = 0;
  bool dead = false;
  const int r = lane >> 2, c = lane & 3;       // mma fragment row / column group
  const int mi = lane >> 3, rr = lane & 7;     // ldmatrix: matrix index, row in matrix
  const int krow = ((mi & 1) << 3) + rr;       // K tile row (token) this lane addresses
  const int vrow = ((mi >> 1) << 3) + rr;      // V tile row (token) this lane addresses
  uint8_t* my_stages = stages + warp * kR * kStageBytes;
  uint64_t* my_bars = bars + warp * kR;

  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    // ---- decode the item
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_start[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int rel = item - s_start[b];
    const int split = rel / Hkv, h = rel - split * Hkv;
    const int nv = s_nv[b];
    const int nsplit = max(1, (nv + SP - 1) / SP);
    const Geom ge = make_geom(s_t[b], p.mode, p.sinks, p.window, p.max_pages, true);
    const int v0 = split * SP, v1 = min(v0 + SP, nv);
    const int cw = (v1 - v0 - warp > 0) ? (v1 - v0 - warp + kW - 1) / kW : 0;
    const int* ptab = p.page_table + (size_t)b * p.max_pages;

    // ---- query fragments (B operand of S = K Q^T): head n = r of the group, dims 2c, 2c+1
    uint32_t qf[8][2];
    {
      const int n = r;
      if (n < g) {
        const uint32_t* qrow = p.q + ((size_t)b * p.Hq + h * g + n) * 64;
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

    auto issue = [&](int k) {
      const int v = v0 + warp + k * kW;
      const int lp = geom_page(ge, v);
      const uint32_t st = issued % kR;
      if (lane == 0) {
        const int phys = ptab[lp];
        uint64_t* bar = my_bars + st;
        if (phys >= 0 && (int64_t)phys < p.n_pool_pages) {
          uint8_t* dst = my_stages + st * kStageBytes;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(bar, kStageBytes);
          const int y = (phys * Hkv + h) * kPageTok;
          tma_load_2d(dst, &tmK, 0, y, bar);
          tma_load_2d(dst + 2048, &tmK, 64, y, bar);
          tma_load_2d(dst + 4096, &tmV, 0, y, bar);
          tma_load_2d(dst + 6144, &tmV, 64, y, bar);
        } else {
          atomicOr(p.err, ODA_DEVERR_PAGE_RANGE);
          mbar_arrive(bar);
        }
      }
      ++issued;
    };

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    if (!dead) {
      __syncwarp();
      const int pre = min(cw, kR);
      for (int k = 0; k < pre; ++k) issue(k);
      for (int k = 0; k < cw; ++k) {
        const uint32_t st = consumed % kR;
        if (!mbar_wait_bounded(my_bars + st, (consumed / kR) & 1u, kWaitNs)) {
          if (lane == 0) atomicOr(p.err, ODA_DEVERR_WAIT_TIMEOUT);
          dead = true;
          break;
        }
        const int v = v0 + warp + k * kW;
        const int lp = geom_page(ge, v);
        const int phys = ptab[lp];
        const bool page_ok = phys >= 0 && (int64_t)phys < p.n_pool_pages;
        const int j0 = lp * kPageTok + r, j1 = j0 + 8;
        const bool in0 = page_ok && geom_has(ge, j0);
        const bool in1 = page_ok && geom_has(ge, j1);
        if (__any_sync(0xffffffffu, in0 || in1)) {
          const uint32_t sb = smem_u32(my_stages + st * kStageBytes);
          // S[token][head] = K[token] . Q[head]
          float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int chunk = 2 * kk + (mi >> 1);
            uint32_t a[4];
            ldsm_x4(a, sb + (chunk >> 3) * 2048 + krow * 128 + (((chunk & 7) ^ rr) << 4));
            mma_bf16_16816(sacc, a, qf[kk][0], qf[kk][1]);
          }
          const float x0 = in0 ? sacc[0] * p.scale_log2 : -INFINITY;
          const float x1 = in0 ? sacc[1] * p.scale_log2 : -INFINITY;
          const float x2 = in1 ? sacc[2] * p.scale_log2 : -INFINITY;
          const float x3 = in1 ? sacc[3] * p.scale_log2 : -INFINITY;
          float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
          const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
          m0 = mn0;
          m1 = mn1;
          l0 *= al0;
          l1 *= al1;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
          }
          const float p0 = exp2f(x0 - mn0), p1 = exp2f(x1 - mn1);
          const float p2 = exp2f(x2 - mn0), p3 = exp2f(x3 - mn1);
          l0 += p0 + p2;
          l1 += p1 + p3;
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
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const int chunk = 2 * mt + (mi & 1);
            uint32_t a[4];
            ldsm_x4_trans(a, sb + 4096 + (chunk >> 3) * 2048 + vrow * 128 +
                                 (((chunk & 7) ^ rr) << 4));
            mma_bf16_16816(o[mt], a, bh0, bh1);
            mma_bf16_16816(o[mt], a, bl0, bl1);
          }
        }
        ++consumed;
        __syncwarp();
        if (k + kR < cw) issue(k + kR);
      }
    }

    // ---- column sums of l across the 8 token rows held by lanes with the same c
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    // ---- this warp's state -> its own (now idle) stage memory
    {
      float* mo = reinterpret_cast<float*>(my_stages);
      float* ml = mo + 8 * kMergeStride;
      const int n0 = 2 * c, n1 = 2 * c + 1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int d = 16 * mt + r;
        if (n0 < g) {
          mo[n0 * kMergeStride + d] = o[mt][0];
          mo[n0 * kMergeStride + d + 8] = o[mt][2];
        }
        if (n1 < g) {
          mo[n1 * kMergeStride + d] = o[mt][1];
          mo[n1 * kMergeStride + d + 8] = o[mt][3];
        }
      }
      if (r == 0) {
        ml[n0 * 2] = m0;
        ml[n0 * 2 + 1] = l0;
        ml[n1 * 2] = m1;
        ml[n1 * 2 + 1] = l1;
      }
    }
    __syncthreads();
    // ---- merge the warps into one partial per query head of the group
    for (int idx = tid; idx < g * 128; idx += kThreads) {
      const int n = idx >> 7, d = idx & 127;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kW; ++w) {
        const float* ml = reinterpret_cast<const float*>(stages + w * kR * kStageBytes) +
                          8 * kMergeStride;
        M = fmaxf(M, ml[n * 2]);
      }
      float O = 0.f, L = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kW; ++w) {
          const float* mo = reinterpret_cast<const float*>(stages + w * kR * kStageBytes);
          const float* ml = mo + 8 * kMergeStride;
          const float mw = ml[n * 2];
          if (mw != -INFINITY) {
            const float s = exp2f(mw - M);
            O += s * mo[n * kMergeStride + d];
            L += s * ml[n * 2 + 1];
          }
        }
      }
      const size_t pi = (size_t)(b * p.Hq + h * g + n) * p.max_splits + split;
      p.part_o[pi * 128 + d] = O;
      if (d == 0) {
        p.part_ml[pi * 2] = M;
        p.part_ml[pi * 2 + 1] = L;
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int old = atomicAdd(&p.counters[b * Hkv + h], 1);
      s_last = (old == nsplit - 1);
    }
    __syncthreads();
    if (s_last) {
      // ---- last CTA of (b, h): merge all splits and the staged current token
      __threadfence();
      float* s_w = reinterpret_cast<float*>(stages);  // [g][nsplit] split weights
      for (int n = warp; n < g; n += kW) {
        const uint32_t* qrow = p.q + ((size_t)b * p.Hq + h * g + n) * 64;
        const uint32_t* krow_new = p.k_new + ((size_t)b * Hkv + h) * 64;
        float acc = 0.f;
        for (int i = lane; i < 64; i += 32) {
          const uint32_t qa = qrow[i], ka = krow_new[i];
          acc += bf16_lo_to_f32(qa) * bf16_lo_to_f32(ka) + bf16_hi_to_f32(qa) * bf16_hi_to_f32(ka);
        }
        const float snew = warp_sum(acc) * p.scale_log2;
        const float* pml = p.part_ml + (size_t)(b * p.Hq + h * g + n) * p.max_splits * 2;
        float M = snew;
        for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, __ldcg(pml + 2 * s));
        M = warp_max(M);
        float L = 0.f;
        for (int s = lane; s < nsplit; s += 32) {
          const float ms = __ldcg(pml + 2 * s);
          const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
          s_w[n * nsplit + s] = w;
          L += w * __ldcg(pml + 2 * s + 1);
        }
        L = warp_sum(L);
        const float wnew = exp2f(snew - M);
        if (lane == 0) {
          s_L[n] = L + wnew;
          s_wnew[n] = wnew;
        }
      }
      __syncthreads();
      for (int idx = tid; idx < g * 128; idx += kThreads) {
        const int n = idx >> 7, d = idx & 127;
        const float* po = p.part_o + (size_t)(b * p.Hq + h * g + n) * p.max_splits * 128 + d;
        const float* wn = s_w + n * nsplit;
        float O0 = 0.f, O1 = 0.f, O2 = 0.f, O3 = 0.f;
        int s = 0;
        for (; s + 4 <= nsplit; s += 4) {
          O0 += wn[s] * __ldcg(po + (size_t)s * 128);
          O1 += wn[s + 1] * __ldcg(po + (size_t)(s + 1) * 128);
          O2 += wn[s + 2] * __ldcg(po + (size_t)(s + 2) * 128);
          O3 += wn[s + 3] * __ldcg(po + (size_t)(s + 3) * 128);
        }
        for (; s < nsplit; ++s) O0 += wn[s] * __ldcg(po + (size_t)s * 128);
        const uint32_t vv = p.v_new[((size_t)b * Hkv + h) * 64 + (d >> 1)];
        const float vd = (d & 1) ? bf16_hi_to_f32(vv) : bf16_lo_to_f32(vv);
        const float O = (O0 + O1) + (O2 + O3) + s_wnew[n] * vd;
        p.out[((size_t)b * p.Hq + h * g + n) * 128 + d] = O / s_L[n];
      }
      if (tid == 0) p.counters[b * Hkv + h] = 0;
    }
    // the stage memory was used through the generic proxy above; the next item's TMA writes
    // it through the async proxy
    fence_proxy_async_smem();
    __syncthreads();
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

// Tensor map over one layer's pool seen as a 2-D array [n_pages*Hkv*16 rows][128 bf16],
// boxes of 16 rows x 64 columns (128 bytes) with the 128-byte swizzle.
oda_status encode_pool(CUtensorMap* m, void* base, int64_t n_pages, int Hkv) {
  EncodeFn enc = get_encode();
  if (!enc) return set_error(ODA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {128, (cuuint64_t)n_pages * Hkv * kPageTok};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, kPageTok};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(ODA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ODA_OK;
}

}  // namespace

int attention_smem_bytes() { return kSmemBytes; }
int attention_threads() { return kThreads; }
int attention_ctas_per_sm() { return kCtasPerSm; }

oda_status launch_attention(oda_ctx* ctx, const oda_kv_layer* layer, const int32_t* page_table,
                            const int32_t* pos, const int32_t* flag, const void* q,
                            const void* k_new, const void* v_new, float* out, int mode,
                            cudaStream_t stream) {
  const oda_config& cf = ctx->cfg;
  if (!layer || !layer->k || !layer->v || !page_table || !pos || !q || !k_new || !v_new || !out ||
      (mode == 1 && !flag))
    return set_error(ODA_ERR_INVALID_ARG, "attention: null pointer argument");
  if (layer->n_pages <= 0 || layer->n_pages * (int64_t)cf.n_kv_heads * kPageTok > INT32_MAX)
    return set_error(ODA_ERR_INVALID_ARG, "attention: n_pages out of range (%lld)",
                     (long long)layer->n_pages);
  if ((reinterpret_cast<uintptr_t>(layer->k) | reinterpret_cast<uintptr_t>(layer->v)) & 15)
    return set_error(ODA_ERR_INVALID_ARG, "attention: K/V pools must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_new) |
       reinterpret_cast<uintptr_t>(v_new) | reinterpret_cast<uintptr_t>(out)) & 3)
    return set_error(ODA_ERR_INVALID_ARG, "attention: q/k_new/v_new/out must be 4-byte aligned");
  CUtensorMap tmK, tmV;
  oda_status st = encode_pool(&tmK, layer->k, layer->n_pages, cf.n_kv_heads);
  if (st != ODA_OK) return st;
  st = encode_pool(&tmV, layer->v, layer->n_pages, cf.n_kv_heads);
  if (st != ODA_OK) return st;
  AttnParams p;
  p.page_table = page_table;
  p.pos = pos;
  p.flag = flag;
  p.q = static_cast<const uint32_t*>(q);
  p.k_new = static_cast<const uint32_t*>(k_new);
  p.v_new = static_cast<const uint32_t*>(v_new);
  p.out = out;
  p.part_o = ctx->part_o;
  p.part_ml = ctx->part_ml;
  p.counters = ctx->attn_cnt;
  p.err = ctx->err;
  p.n_pool_pages = layer->n_pages;
  p.B = cf.batch;
  p.Hq = cf.n_q_heads;
  p.Hkv = cf.n_kv_heads;
  p.g = ctx->g;
  p.max_pages = cf.max_pages;
  p.max_splits = ctx->max_splits;
  p.sinks = cf.sinks;
  p.window = cf.window;
  p.mode = mode;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  attn_kernel<<<ctx->attn_ctas, kThreads, kSmemBytes, stream>>>(tmK, tmV, p);
  return check_cuda(cudaGetLastError(), "attention launch");
}

oda_status prepare_attention_kernel() {
  return check_cuda(cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes),
                    "cudaFuncSetAttribute(attention)");
}

oda_status launch_index_positions(oda_ctx* ctx, int mode, const int32_t* pos, const int32_t* flag,
                                  int32_t* positions, int32_t cap, int32_t* counts,
                                  cudaStream_t stream) {
  if (!pos || !positions || !counts || cap <= 0 || (mode == 1 && !flag) || (mode != 0 && mode != 1))
    return set_error(ODA_ERR_INVALID_ARG, "index_positions: bad argument");
  const oda_config& cf = ctx->cfg;
  index_positions_kernel<<<(cf.batch + 31) / 32, 32, 0, stream>>>(
      pos, flag, cf.batch, mode, cf.sinks, cf.window, cf.max_pages, positions, cap, counts);
  return check_cuda(cudaGetLastError(), "index_positions launch");
}

}  // namespace oda
