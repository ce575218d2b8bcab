// Fused S3R sparse draft step in one tcgen05 kernel: page scoring from the
// Quest page summaries, top-B selection, and attention over the kept pages
// ("S3R: Fast and Faithful RL Rollouts via Self-Sparse Speculative Decoding",
// weekinpapers.com, Abstract: sparse attention proposes the draft tokens; page
// choice after Quest, on the mlsanity.com page's reference list).
//
// Work: one CTA per piece of a (sequence, KV head) unit. When the units alone
// would leave SMs idle, each unit's kept-page list is cut into `parts` pieces
// whose CTAs form one thread-block cluster: each scores its share of the
// unit's pages, the first CTA selects over all of them (keys gathered through
// distributed shared memory) and hands the list back to the others; each CTA
// attends over its piece of the list and the last to finish merges the
// pieces by log-sum-exp. Launches with more units than SMs take the selection
// kernel and the split-KV attention kernel instead.
//
// Selection of a unit (all 256 threads of the CTA):
//   score(p) = sum_g sum_d max(q_g,d kmin_p,d, q_g,d kmax_p,d) for p < n_b,
//   folded per channel into A max(kmin, kmax) + B min(kmin, kmax) with
//   A = sum_g max(q_g, 0) and B = sum_g min(q_g, 0) (exact in real arithmetic),
//   accumulated in float64; the tail page n_b - 1 is summarised from K itself
//   (its keys change while the sequence decodes). The summary rows (and the
//   tail page's K) are staged by cp.async in the K/V ring, which is still
//   empty, chunk by chunk, and each quarter of a chunk is scored as soon as
//   it lands. The kept pages come from the order-preserving keys: for up to
//   256 pages each page's rank among the keys decides, beyond that a radix
//   select of the budget-th largest key; they go, in ascending order with
//   ties to the lower page, into a list in shared memory.
//
// Attention over the kept pages is the token-major pipeline of s3r_attn_tok.cu
// (S^T = K Q^T and O^T += V^T P^T per 128-token stage, fp32 in TMEM):
// warp 4 streams the listed pages by TMA into the ring, warp 5 issues the
// MMAs, warps 0-3 run the softmax and the epilogue (warps 6-7 only select).
#include <cuda_bf16.h>

#include <cmath>
#include <type_traits>

#include "s3r_attn_common.cuh"
#include "s3r_device.cuh"
#include "s3r_internal.h"
#include "s3r_tok_common.cuh"

namespace s3r {
namespace {

constexpr int kDfThreads = 256;
constexpr int kDfProducer = 4;
constexpr int kDfMma = 5;
constexpr int kDfMaxPages = 1024;              // pages per sequence (keys kept in shared memory)
constexpr int kDfMaxBudget = 128;
constexpr int kDfN = 16;                       // MMA rows: the G <= 8 query heads, padded
constexpr int kDfNR = 8;                       // softmax rows
constexpr int kBarAll = 2;                     // named barrier of the selection (all threads)

template <int D>
struct DfLay {
  using T = TokLay<kDfN, D>;
  static constexpr int kNS = T::kNS;
  static constexpr uint32_t kRing = kNS * 2 * T::kTileBytes;
  static constexpr uint32_t kRowBytes = 2 * D * 2;                 // kmin and kmax rows of one page
  static constexpr uint32_t kTailBytes = 64 * D * 2;               // K of one page (P <= 64)
  static constexpr int kChunkPages = (int)((kRing - kTailBytes) / kRowBytes);
  static constexpr uint32_t kOffKeys = T::kOffKV + kRing;          // u64 [kDfMaxPages]
  static constexpr uint32_t kOffPhys = kOffKeys + 8 * kDfMaxPages; // int [kDfMaxPages]
  static constexpr uint32_t kOffList = kOffPhys + 4 * kDfMaxPages; // int2 [kDfMaxBudget]
  static constexpr uint32_t kOffAB = kOffList + 8 * kDfMaxBudget;  // double [2][D]
  static constexpr uint32_t kOffTail = kOffAB + 2 * 8 * D;         // bf16 [2][D]
  static constexpr uint32_t kOffHist = kOffTail + 2 * 2 * D;       // u32 [256]
  static constexpr uint32_t kDynBytes = kOffHist + 4 * 256;
  static_assert(kChunkPages >= 64, "staging chunk");
  static_assert(8 * kDfMaxPages >= kDfThreads * 16, "tail scratch fits in the key array");
  static_assert(12 * 8 * kDfMaxBudget <= kRing, "candidate arrays fit in the ring");
};

__device__ __forceinline__ void grp_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Whether `pred` holds on every thread of the group (a barrier of its own):
// turns per-thread outcomes of bounded waits into one decision.
__device__ __forceinline__ bool grp_all(bool pred, int id, int n) {
  int r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
               "selp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((int)pred), "r"(id), "r"(n) : "memory");
  return r != 0;
}

__device__ __forceinline__ unsigned long long order_key(double x) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// bf16 pair (low half first) as floats
__device__ __forceinline__ void bf2(uint32_t u, float& a, float& b) {
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xFFFF0000u);
}

// One work item: piece k of unit u = b * Hkv + h.
struct DItem {
  int u, k, b, h, L, n_b, npg, k0;
  bool bad;
};
__device__ __forceinline__ DItem draft_item(const AttnParams& p, int it) {
  DItem d;
  d.u = it / p.parts;
  d.k = it - d.u * p.parts;
  d.b = d.u / p.Hkv;
  d.h = d.u - d.b * p.Hkv;
  d.L = __ldg(p.context_lens + d.b);
  d.bad = d.L < 1 || d.L > p.max_pages * p.P;
  d.n_b = d.bad ? 0 : (d.L + p.P - 1) / p.P;
  const int n_sel = min(p.budget, d.n_b);
  d.k0 = d.k * n_sel / p.parts;
  d.npg = (d.k + 1) * n_sel / p.parts - d.k0;
  return d;
}

struct SelSmem {
  unsigned long long* keys;   // [kDfMaxPages]
  int* phys;                  // [kDfMaxPages] physical ids of the unit's pages
  double* ab;                 // [2][D] the folded query weights A, B
  __nv_bfloat16* tail;        // [2][D] min / max of the tail page
  unsigned* hist;             // [256]
};
struct SelScratch {
  unsigned long long kred[2][8];
  unsigned long long prefix;
  int k, done, shift, start;
  int wsum[8];
};

// Exclusive prefix sum over the group's nthr threads (whole warps); *total
// receives the sum.
__device__ int grp_exclusive_scan(int v, int tg, int nthr, int barid, SelScratch& sc, int* total) {
  const int lane = tg & 31, gw = tg >> 5, nw = nthr >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sc.wsum[gw] = x;
  grp_sync(barid, nthr);
  if (gw == 0) {
    int w = lane < nw ? sc.wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sc.wsum[lane] = w;              // inclusive
  }
  grp_sync(barid, nthr);
  const int before = (gw > 0 ? sc.wsum[gw - 1] : 0) + x - v;
  *total = sc.wsum[nw - 1];
  grp_sync(barid, nthr);
  return before;
}

// Inputs of a unit's selection that no kernel of the library writes (so they
// may be read before the grid-dependency wait): the physical ids of its pages
// and the folded query weights of its KV head.
template <int D>
__device__ void sel_prepare(const AttnParams& p, const DItem& d, int tg, int nthr, const SelSmem& sm) {
  if (d.bad) return;
  const int32_t* bt = p.block_table + (size_t)d.b * p.max_pages;
  for (int i = tg; i < d.n_b; i += nthr) sm.phys[i] = __ldg(bt + i);
  if (d.n_b <= p.budget) return;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)d.b * p.Hq + (size_t)d.h * p.G) * D;
  for (int c = tg; c < D; c += nthr) {
    float v[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) v[g] = g < p.G ? __bfloat162float(q[(size_t)g * D + c]) : 0.f;   // all in flight
    double a = 0.0, z = 0.0;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const double x = static_cast<double>(v[g]);
      if (x > 0.0) a += x; else z += x;                  // zero padding adds nothing
    }
    sm.ab[c] = a;
    sm.ab[D + c] = z;
  }
}

// Scores of pages [g0, g1) (none of them the tail page) into sm.keys; the
// rows of page pg sit at rows + (pg - c0) * kRowBytes (kmin row, then kmax).
// Sixteen pages per warp and round, each lane holding D / 32 channels of
// every page; the sixteen page sums are reduced across the warp together
// (halving exchanges: lane l ends with page l % 16), which keeps sixteen
// independent chains in flight per lane.
template <int D>
__device__ void score_pages(const AttnParams& p, int c0, int g0, int g1, const uint8_t* rows, int tg, int nthr,
                            const SelSmem& sm) {
  constexpr int CPL = D / 32;
  constexpr int kU = 16;
  using Raw = typename std::conditional<CPL == 4, uint2, uint32_t>::type;
  const int lane = tg & 31, gw = tg >> 5, nw = nthr >> 5;
  double wa[CPL], wb[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) { wa[c] = sm.ab[lane * CPL + c]; wb[c] = sm.ab[D + lane * CPL + c]; }
  for (int pg0 = g0 + gw * kU; pg0 < g1; pg0 += nw * kU) {
    Raw lo[kU], hi[kU];
    bool ok[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int pg = pg0 + u;
      const int ph = pg < g1 ? sm.phys[pg] : -1;
      ok[u] = ph >= 0 && ph < p.num_pages_total;
      const Raw* r = reinterpret_cast<const Raw*>(rows + (size_t)(pg - c0) * DfLay<D>::kRowBytes) + lane;
      if (ok[u]) { lo[u] = r[0]; hi[u] = r[32]; }      // kmin row, kmax row (2 D bytes apart)
    }
    double acc[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      double s0 = 0.0, s1 = 0.0;
      if (ok[u]) {
        uint32_t lw[CPL / 2], hw[CPL / 2];
        if constexpr (CPL == 4) { lw[0] = ((uint2&)lo[u]).x; lw[1] = ((uint2&)lo[u]).y; hw[0] = ((uint2&)hi[u]).x; hw[1] = ((uint2&)hi[u]).y; }
        else { lw[0] = (uint32_t&)lo[u]; hw[0] = (uint32_t&)hi[u]; }
#pragma unroll
        for (int w = 0; w < CPL / 2; ++w) {
          float l0, l1, r0, r1;
          bf2(lw[w], l0, l1);
          bf2(hw[w], r0, r1);
          s0 = fma(wa[2 * w], static_cast<double>(fmaxf(l0, r0)), s0);
          s1 = fma(wb[2 * w], static_cast<double>(fminf(l0, r0)), s1);
          s0 = fma(wa[2 * w + 1], static_cast<double>(fmaxf(l1, r1)), s0);
          s1 = fma(wb[2 * w + 1], static_cast<double>(fminf(l1, r1)), s1);
        }
      }
      acc[u] = s0 + s1;
    }
#pragma unroll
    for (int w = kU / 2; w >= 1; w >>= 1) {
      const bool up = (lane & w) != 0;
#pragma unroll
      for (int k = 0; k < w; ++k) {
        const double send = up ? acc[k] : acc[k + w];
        const double keep = up ? acc[k + w] : acc[k];
        acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, w);
      }
    }
    const double v = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 16);
    const int pg = pg0 + (lane & 15);
    if (lane < kU && pg < g1) {
      bool okp = false;
#pragma unroll
      for (int u = 0; u < kU; ++u) okp = (u == lane) ? ok[u] : okp;
      if (!okp) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      sm.keys[pg] = okp ? order_key(v) : 0ull;
    }
  }
}

// Min and max of the tail page's valid tokens per channel into sm.tail (bf16,
// exact). src: the page's K rows (shared or global memory). Thread = channel
// pair x token group; the groups merge through `scratch` (float4 [ngrp][D/2]).
template <int D>
__device__ void tail_minmax(const __nv_bfloat16* src, int valid, int tg, int nthr, int barid, const SelSmem& sm,
                            float4* scratch) {
  constexpr int CP = D / 2;
  const int cp = tg % CP, tq = tg / CP, ngrp = nthr / CP;
  float mn0 = INFINITY, mn1 = INFINITY, mx0 = -INFINITY, mx1 = -INFINITY;
  for (int t = tq; t < valid; t += ngrp) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(src + (size_t)t * D + 2 * cp);
    float a, b;
    bf2(u, a, b);
    mn0 = fminf(mn0, a); mx0 = fmaxf(mx0, a);
    mn1 = fminf(mn1, b); mx1 = fmaxf(mx1, b);
  }
  if (ngrp > 1) {
    scratch[tq * CP + cp] = make_float4(mn0, mn1, mx0, mx1);
    grp_sync(barid, nthr);
    if (tg < CP) {
      for (int g = 1; g < ngrp; ++g) {
        const float4 o = scratch[g * CP + cp];
        mn0 = fminf(mn0, o.x); mn1 = fminf(mn1, o.y); mx0 = fmaxf(mx0, o.z); mx1 = fmaxf(mx1, o.w);
      }
    }
  }
  if (tg < CP) {
    sm.tail[2 * cp] = __float2bfloat16_rn(mn0);
    sm.tail[2 * cp + 1] = __float2bfloat16_rn(mn1);
    sm.tail[D + 2 * cp] = __float2bfloat16_rn(mx0);
    sm.tail[D + 2 * cp + 1] = __float2bfloat16_rn(mx1);
  }
}

// Rank of key kp (page i) among keys[0..n): the keys above it, plus the
// equal keys of lower pages (ties go to the lower page). keys is 8-byte
// aligned; one key is taken alone when that puts the rest on a 16-byte
// boundary, then pairs of keys by 16-byte broadcast reads, four pairs per
// step with separate counters.
__device__ __forceinline__ int key_rank(const unsigned long long* keys, int n, unsigned long long kp, int i) {
  int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
  int q = 0;
  if ((reinterpret_cast<uintptr_t>(keys) & 15u) != 0 && n > 0) {
    r0 += (keys[0] > kp) + (keys[0] == kp && 0 < i);
    q = 1;
  }
  const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys + q);   // 16-byte aligned
  for (int j = 0; q + 8 <= n; q += 8, j += 4) {
    const ulonglong2 a = k2[j], b = k2[j + 1], c = k2[j + 2], e = k2[j + 3];
    r0 += (a.x > kp) + (a.x == kp && q < i) + (a.y > kp) + (a.y == kp && q + 1 < i);
    r1 += (b.x > kp) + (b.x == kp && q + 2 < i) + (b.y > kp) + (b.y == kp && q + 3 < i);
    r2 += (c.x > kp) + (c.x == kp && q + 4 < i) + (c.y > kp) + (c.y == kp && q + 5 < i);
    r3 += (e.x > kp) + (e.x == kp && q + 6 < i) + (e.y > kp) + (e.y == kp && q + 7 < i);
  }
  for (; q < n; ++q) r0 += (keys[q] > kp) + (keys[q] == kp && q < i);
  return (r0 + r1) + (r2 + r3);
}

// Candidates of one group of at most nthr pages page0.. (keys in page
// order): the pages whose rank in the group is below `budget`, appended in
// page order to cand_key / cand_page at `base`. Returns the number appended.
__device__ int group_candidates(const unsigned long long* keys, int page0, int n, int budget,
                                unsigned long long* cand_key, int* cand_page, int base, int tg, int nthr,
                                int barid, SelScratch& sc) {
  bool keep = false;
  unsigned long long kp = 0;
  if (tg < n) {
    kp = keys[tg];
    keep = key_rank(keys, n, kp, tg) < budget;
  }
  int tot;
  const int pos = grp_exclusive_scan(keep ? 1 : 0, tg, nthr, barid, sc, &tot);
  if (keep) {
    cand_key[base + pos] = kp;
    cand_page[base + pos] = page0 + tg;
  }
  return tot;
}

// The kept pages of item d's unit, ascending, into `list` (logical,
// physical) and, for the unit's first piece, into p.selected_out. All
// threads of the CTA, after sel_prepare and the grid-dependency wait.
// clustered: the unit is shared by the p.parts CTAs of this cluster (rank =
// d.k); each scores its share of the pages and sends its candidates (the
// pages that are top-B within their group of at most 256) to the first CTA,
// which ranks the candidates and hands the list back. The global top-B is
// contained in the union of the groups' top-B, so the result is exact.
template <int D>
__device__ void select_unit(const AttnParams& p, const DItem& d, int2* list, const SelSmem& sm, SelScratch& sc,
                            uint8_t* stage, uint32_t bar_g0, uint32_t bar_g1, bool clustered, volatile int* abort) {
  using Lay = DfLay<D>;
  constexpr int nthr = kDfThreads, barid = kBarAll;
  const int tg = threadIdx.x, lane = tg & 31, gw = tg >> 5;
  const bool write_out = d.k == 0;
  int32_t* out = p.selected_out + ((size_t)d.b * p.Hkv + d.h) * p.budget;
  for (int k = tg; k < p.budget; k += nthr) list[k] = make_int2(-1, -1);
  if (d.bad) {
    if (write_out) {
      for (int k = tg; k < p.budget; k += nthr) out[k] = -1;
      if (tg == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
    }
    return;
  }
  const int n_b = d.n_b;
  if (n_b <= p.budget) {
    for (int k = tg; k < p.budget; k += nthr) {
      if (k < n_b) list[k] = make_int2(k, sm.phys[k]);
      if (write_out) out[k] = k < n_b ? k : -1;
    }
    return;
  }
  // this CTA's share of the pages
  const int parts = clustered ? p.parts : 1, rank = clustered ? d.k : 0;
  const int s0 = rank * n_b / parts, s1 = (rank + 1) * n_b / parts;
  const int tail = n_b - 1;
  const bool has_tail = s0 <= tail && tail < s1;
  const int valid = d.L - tail * p.P;
  const int tail_ph = sm.phys[tail];
  const bool tail_ok = tail_ph >= 0 && tail_ph < p.num_pages_total;
  const __nv_bfloat16* tail_src =
      static_cast<const __nv_bfloat16*>(p.k_cache) + ((size_t)tail_ph * p.Hkv + d.h) * p.P * D;
  const __nv_bfloat16* kmn = static_cast<const __nv_bfloat16*>(p.kmin);
  const __nv_bfloat16* kmx = static_cast<const __nv_bfloat16*>(p.kmax);
  float4* scratch = reinterpret_cast<float4*>(sm.keys);
  uint8_t* rows = stage + Lay::kTailBytes;
  bool ok = true;
  // summary rows of the share's pages, bulk-copied into the empty ring chunk
  // by chunk, each chunk in two halves on two barriers so that the first
  // half is scored while the second is still landing; the tail page's K
  // (when in the share) with the first half of the first chunk
  const int e = min(s1, tail);                           // the share's pages other than the tail
  int phase = 0;
  for (int c0 = s0, first = 1; first || c0 < e; c0 += Lay::kChunkPages, first = 0, ++phase) {
    const int c1 = max(c0, min(e, c0 + Lay::kChunkPages));
    const int mid = c0 + (c1 - c0 + 1) / 2;
    if (first && has_tail && tail_ok && tg == 0) {
      const uint32_t bytes = (uint32_t)valid * D * 2;
      mbar_expect_tx(bar_g0, bytes);
      bulk_load(smem_addr(stage), tail_src, bytes, bar_g0);
    }
    for (int pg = c0 + tg; pg < c1; pg += nthr) {
      const int ph = sm.phys[pg];
      if (ph < 0 || ph >= p.num_pages_total) continue;
      const uint32_t bar = pg < mid ? bar_g0 : bar_g1;
      const size_t base = ((size_t)ph * p.Hkv + d.h) * D;
      const uint32_t dst = smem_addr(rows + (size_t)(pg - c0) * Lay::kRowBytes);
      mbar_expect_tx(bar, 4u * D);
      bulk_load(dst, kmn + base, 2u * D, bar);
      bulk_load(dst + 2u * D, kmx + base, 2u * D, bar);
    }
    grp_sync(barid, nthr);                               // every expectation is registered
    if (tg == 0) { mbar_arrive(bar_g0); mbar_arrive(bar_g1); }
    ok = ok && grp_all(mbar_wait(bar_g0, (uint32_t)(phase & 1), abort, p.status), barid, nthr);
    if (ok && first && has_tail && tail_ok) {
      tail_minmax<D>(reinterpret_cast<const __nv_bfloat16*>(stage), valid, tg, nthr, barid, sm, scratch);
      grp_sync(barid, nthr);                             // the scratch is the key array
    }
    if (ok) score_pages<D>(p, c0, c0, mid, rows, tg, nthr, sm);
    ok = ok && grp_all(mbar_wait(bar_g1, (uint32_t)(phase & 1), abort, p.status), barid, nthr);
    if (ok) score_pages<D>(p, c0, mid, c1, rows, tg, nthr, sm);
    fence_proxy_async_smem();                            // reads of the staged rows before copies reuse them
    grp_sync(barid, nthr);
    if (!ok) break;
  }
  // the tail page, scored from its fresh min / max (first warp)
  if (ok && has_tail && gw == 0) {
    constexpr int CPL = D / 32;
    double a0 = 0.0, a1 = 0.0;
    if (tail_ok) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int ch = lane * CPL + c;
        const float l = __bfloat162float(sm.tail[ch]), r = __bfloat162float(sm.tail[D + ch]);
        a0 = fma(sm.ab[ch], static_cast<double>(fmaxf(l, r)), a0);
        a1 = fma(sm.ab[D + ch], static_cast<double>(fminf(l, r)), a1);
      }
    }
    double v = a0 + a1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      if (!tail_ok) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      sm.keys[tail] = tail_ok ? order_key(v) : 0ull;
    }
  }
  grp_sync(barid, nthr);
  // ---- candidates: the top-B of each group of at most nthr pages of the
  // share, in page order, at their place in the first CTA's candidate array
  // (the stage's first bytes: the ring is idle until the list is done)
  unsigned long long* cand_key = reinterpret_cast<unsigned long long*>(stage);     // [8 * kDfMaxBudget]
  int* cand_page = reinterpret_cast<int*>(stage + 8 * 8 * kDfMaxBudget);            // [8 * kDfMaxBudget]
  auto cands_of = [&](int lo, int hi) {                  // candidates of pages [lo, hi), whole groups
    int c = 0;
    for (int g = lo; g < hi; g += nthr) c += min(p.budget, min(hi, g + nthr) - g);
    return c;
  };
  if (clustered) cluster_sync_all();                     // every CTA scored: the first one's stage is free
  int base = 0;
  for (int r = 0; r < rank; ++r) base += cands_of(r * n_b / parts, (r + 1) * n_b / parts);
  if (ok) {
    for (int g = s0; g < s1; g += nthr) {
      // this group's candidates into this CTA's own array, then (other CTAs
      // of a cluster) copied to the first CTA's
      const int n = min(s1, g + nthr) - g;
      const int got = group_candidates(sm.keys + g, g, n, p.budget, cand_key, cand_page, base, tg, nthr, barid, sc);
      grp_sync(barid, nthr);
      if (clustered && rank != 0)
        for (int k = tg; k < got; k += nthr) {
          st_cluster_u64(&cand_key[base + k], 0u, cand_key[base + k]);
          st_cluster_u32(&cand_page[base + k], 0u, (uint32_t)cand_page[base + k]);
        }
      base += got;
    }
  }
  if (clustered) cluster_sync_all();                     // all candidates are in the first CTA
  if (rank == 0 && ok) {
    // ---- final rank among the candidates (ascending page order already)
    int nc = 0;                                          // candidates of every share
    for (int r = 0; r < parts; ++r) nc += cands_of(r * n_b / parts, (r + 1) * n_b / parts);
    int kept_before = 0;
    for (int c = 0; c < nc; c += nthr) {
      const int i = c + tg;
      bool keep = false;
      if (i < nc) keep = key_rank(cand_key, nc, cand_key[i], i) < p.budget;
      int tot;
      const int pos = kept_before + grp_exclusive_scan(keep ? 1 : 0, tg, nthr, barid, sc, &tot);
      if (keep && pos < p.budget) {
        const int pg = cand_page[i];
        list[pos] = make_int2(pg, sm.phys[pg]);
        if (write_out) out[pos] = pg;
      }
      kept_before += tot;
    }
    grp_sync(barid, nthr);
  }
  if (clustered) {
    // hand the list to the other pieces' CTAs
    grp_sync(barid, nthr);
    if (rank == 0)
      for (int r = 1; r < parts; ++r)
        for (int k = tg; k < p.budget; k += nthr)
          st_cluster_u64(&list[k], (uint32_t)r, *reinterpret_cast<const unsigned long long*>(&list[k]));
    cluster_sync_all();
  }
}

// Stage cursor of the MMA issuer over the CTA's items with pages.
struct DCur {
  int it, j, nst, g, s;
  bool valid;
  int b, h;
};
__device__ __forceinline__ void dcur_seek(const AttnParams& p, int it1, int ppt, DCur& c) {
  while (c.it < it1) {
    const DItem d = draft_item(p, c.it);
    if (d.npg > 0) {
      c.nst = (d.npg + ppt - 1) / ppt;
      c.b = d.b;
      c.h = d.h;
      c.valid = true;
      return;
    }
    ++c.it;
  }
  c.valid = false;
}
__device__ __forceinline__ void dcur_next(const AttnParams& p, int it1, int ppt, DCur& c) {
  ++c.g;
  if (++c.j >= c.nst) {
    c.j = 0;
    ++c.s;
    ++c.it;
    dcur_seek(p, it1, ppt, c);
  }
}

template <int D>
__global__ void __launch_bounds__(kDfThreads, 1)
draft_fused_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const AttnParams p) {
  using Lay = DfLay<D>;
  using L = TokLay<kDfN, D>;
  constexpr int N = kDfN, NR = kDfNR, NS = L::kNS;
  extern __shared__ __align__(1024) uint8_t dyn_raw[];
  uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t s_bar[2 * NS + 10];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_ticket;
  __shared__ int s_stage_lp[NS][8];
  __shared__ float s_red[4][64];
  __shared__ float s_mx[64];
  __shared__ __align__(16) float s_nu[64];
  __shared__ __align__(16) float s_alpha[64];
  __shared__ SelScratch s_sc;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();

  // one item per CTA: piece blockIdx.x % parts (the CTA's rank in its
  // cluster) of unit blockIdx.x / parts
  const int it0 = blockIdx.x, it1 = blockIdx.x + 1;
  const int ppt = kTok / p.P;                             // pages per stage

  const uint32_t bar0 = smem_addr(&s_bar[0]);
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const int B_FULL = 0, B_EMPTY = NS, B_SFULL = 2 * NS, B_PFULL = 2 * NS + 2, B_ODONE = 2 * NS + 4,
            B_QFULL = 2 * NS + 6, B_TD = 2 * NS + 7, B_G0 = 2 * NS + 8, B_G1 = 2 * NS + 9;
  constexpr int PB = L::kPBufs;
  uint8_t* sQ = dyn;
  uint8_t* sP = dyn + L::kOffP;
  uint8_t* sKV = dyn + L::kOffKV;
  const uint32_t aQ = smem_addr(sQ), aP = smem_addr(sP), aKV = smem_addr(sKV);
  SelSmem sm;
  sm.keys = reinterpret_cast<unsigned long long*>(dyn + Lay::kOffKeys);
  sm.phys = reinterpret_cast<int*>(dyn + Lay::kOffPhys);
  sm.ab = reinterpret_cast<double*>(dyn + Lay::kOffAB);
  sm.tail = reinterpret_cast<__nv_bfloat16*>(dyn + Lay::kOffTail);
  sm.hist = reinterpret_cast<unsigned*>(dyn + Lay::kOffHist);
  int2* s_list = reinterpret_cast<int2*>(dyn + Lay::kOffList);   // [kDfMaxBudget]

  if (warp == kDfMma) {
    tmem_alloc(smem_addr(&s_tmem), 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(BAR(B_FULL + i), 1); mbar_init(BAR(B_EMPTY + i), 1); }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SFULL + 1), 1);
    mbar_init(BAR(B_PFULL), 128);
    mbar_init(BAR(B_PFULL + 1), 128);
    mbar_init(BAR(B_ODONE), 1);
    mbar_init(BAR(B_ODONE + 1), 1);
    mbar_init(BAR(B_QFULL), 128);
    mbar_init(BAR(B_TD), 1);
    mbar_init(BAR(B_G0), 1);
    mbar_init(BAR(B_G1), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kDfProducer && lane == 0) { prefetch_tensormap(&tmK); prefetch_tensormap(&tmV); }

  // Softmax threads: the first unit's query rows (an input) into registers.
  constexpr int kQC = L::kQChunks;
  constexpr int kDc = D / 8;                             // 16-byte chunks per Q row
  uint4 qr[kQC];
  auto q_fetch = [&](int b, int h) {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
    const size_t base = (size_t)b * p.Hq + (size_t)h * p.G;
#pragma unroll
    for (int k = 0; k < kQC; ++k) {
      const int ch = tid + 128 * k, r = ch / kDc, c16 = ch - (ch / kDc) * kDc;
      qr[k] = r < p.rows ? __ldg(reinterpret_cast<const uint4*>(q + (base + r) * D + c16 * 8))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  DCur first;
  first.it = it0; first.j = 0; first.g = 0; first.s = 0; first.nst = 0;
  dcur_seek(p, it1, ppt, first);
  if (warp < 4 && first.valid) q_fetch(first.b, first.h);

  // ---- the unit's selection, by every thread, staged through the empty ring
  const DItem d0 = draft_item(p, it0);
  const bool clustered = p.parts > 1 && !d0.bad && d0.n_b > p.budget;   // uniform over the cluster
  sel_prepare<D>(p, d0, tid, kDfThreads, sm);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  pdl_wait();                                            // summaries, outputs and workspace from here on
  select_unit<D>(p, d0, s_list, sm, s_sc, sKV, BAR(B_G0), BAR(B_G1), clustered, &s_abort);
  __syncthreads();

  if (warp == kDfProducer) {
    // ======================================================= producer warp
    const uint64_t pol = l2_policy_evict_first();
    int g = 0;
    bool ok = __all_sync(0xffffffffu, !s_abort);
    for (int it = it0; it < it1 && ok; ++it) {
      const DItem d = d0;                                  // the CTA's one item
      const int2* list = s_list;
      const int nst = (d.npg + ppt - 1) / ppt;
      for (int j = 0; j < nst; ++j, ++g) {
        const int st = g % NS;
        int my_lp = -1, my_ph = -1;
        if (lane < ppt && j * ppt + lane < d.npg) {
          const int2 e = list[d.k0 + j * ppt + lane];
          my_lp = e.x;
          my_ph = e.y;
          if (my_ph < 0 || my_ph >= p.num_pages_total) {
            flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
            my_ph = -1;
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_EMPTY + st), ((g / NS) & 1) ^ 1, &s_abort, p.status))) {
          ok = false;
          break;
        }
        if (lane < 8) s_stage_lp[st][lane] = (lane < ppt && my_ph >= 0) ? my_lp : -1;
        const unsigned real = __ballot_sync(0xffffffffu, my_ph >= 0);
        __syncwarp();
        if (lane == 0)
          mbar_arrive_expect_tx(BAR(B_FULL + st), (uint32_t)__popc(real) * L::kHalves * 2u * (uint32_t)p.P * 128u);
        __syncwarp();
        if (my_ph >= 0) {
          const uint32_t dK = aKV + st * 2 * L::kTileBytes, dV = dK + L::kTileBytes;
          const int z = my_ph * p.Hkv + d.h;
#pragma unroll
          for (int hh = 0; hh < L::kHalves; ++hh) {
            const uint32_t off = hh * (kTok * 128) + lane * (p.P * 128);
            tma_load_3d(dK + off, &tmK, BAR(B_FULL + st), hh * 64, 0, z, pol);
            tma_load_3d(dV + off, &tmV, BAR(B_FULL + st), hh * 64, 0, z, pol);
          }
        }
      }
    }
    if (lane == 0)
      for (int k = max(0, g - NS); k < g; ++k) mbar_wait_drain(BAR(B_FULL + k % NS), (k / NS) & 1, p.status);
  } else if (warp == kDfMma) {
    // ======================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(kTok, N, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(D, N, true, false);
      DCur qc = first;
      DCur pc = first;
      const uint64_t dQ0 = smem_desc_sw128(aQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(aKV, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(aKV + L::kTileBytes, kTok * 128, 1024);
      const uint64_t dP0 = smem_desc_sw128(aP, 16, 1024);
      constexpr uint64_t kQHalf = (N * 128) >> 4, kPHalf = (N * 128) >> 4;
      constexpr uint64_t kStage = (2 * L::kTileBytes) >> 4, kKHalf = (kTok * 128) >> 4, kVStep = (16 * 128) >> 4;
      auto issue_qk = [&]() {
        tc_fence_after();
        const int st = qc.g % NS;
        const uint64_t kd = dK0 + (uint64_t)st * kStage;
        const uint32_t dS = tmem + L::kColS + (qc.g & 1) * N;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(kk & 3) * 2;
          umma_f16(dS, kd + (kk >> 2) * kKHalf + off, dQ0 + (kk >> 2) * kQHalf + off, idQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(BAR(B_SFULL + (qc.g & 1)));
        dcur_next(p, it1, ppt, qc);
      };
      auto issue_pv = [&]() {
        tc_fence_after();
        const int st = pc.g % NS;
        const uint64_t vd = dV0 + (uint64_t)st * kStage;
        const uint32_t tO = tmem + L::kColO;
        const uint32_t acc0 = pc.j > 0 ? 1u : 0u;
        const uint64_t pd = dP0 + (uint64_t)(pc.g % PB) * (L::kPBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk)
          umma_f16(tO, vd + (uint64_t)kk * kVStep, pd + (kk >> 2) * kPHalf + (uint64_t)(kk & 3) * 2, idPV,
                   kk > 0 ? 1u : acc0);
        umma_commit(BAR(B_EMPTY + st));
        umma_commit(BAR(B_ODONE + (pc.g & 1)));
        dcur_next(p, it1, ppt, pc);
      };
      unsigned long long idle_since = 0;
      uint32_t spins = 0;
      while (pc.valid && !s_abort) {
        bool progress = false;
        if (mbar_test_wait(BAR(B_PFULL + (pc.g & 1)), (pc.g >> 1) & 1)) {
          issue_pv();
          progress = true;
        }
        if (qc.valid && qc.g <= pc.g + 1 && (qc.j != 0 || mbar_test_wait(BAR(B_QFULL), qc.s & 1)) &&
            mbar_test_wait(BAR(B_FULL + qc.g % NS), (qc.g / NS) & 1)) {
          issue_qk();
          progress = true;
        }
        if (progress) {
          idle_since = 0;
          continue;
        }
        if ((++spins & 63u) == 0) {
          if (s_abort) break;
          const unsigned long long now = globaltimer_ns();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            s_abort = 1;
            flag_status(p.status, S3R_DEV_WAIT_TIMEOUT);
            break;
          }
        }
      }
      umma_commit(BAR(B_TD));
    }
  } else if (warp < 4) {
    // ======================================================= softmax warps
    // Thread t: token t of each stage (TMEM lane t of S^T), and TMEM lane t
    // of O^T in the epilogue (dimension t for D = 128; for D = 64 the M = 64
    // accumulator puts dimension 16q + l in lane 32q + l, l < 16).
    const int q4 = warp;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int d_mine = (D == 128) ? tid : (lane < 16 ? 16 * q4 + lane : -1);
    const int log2P = __ffs(p.P) - 1;
    const float c = p.scale_log2;
    auto q_store = [&]() {
#pragma unroll
      for (int k = 0; k < kQC; ++k) {
        const int ch = tid + 128 * k, r = ch / kDc, c16 = ch - (ch / kDc) * kDc;
        *reinterpret_cast<uint4*>(sQ + (c16 >> 3) * (N * 128) + r * 128 + (((c16 & 7) ^ (r & 7)) << 4)) = qr[k];
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(B_QFULL));
    };
    if (first.valid) q_store();
    {
      // P rows NR..N-1 (padding) are zero in both buffers for the whole run
      const int half = tid >> 6, tt = tid & 63, ck = tt >> 3;
#pragma unroll
      for (int b2 = 0; b2 < PB; ++b2) {
        uint8_t* pb = sP + b2 * L::kPBytes + half * (N * 128) + (tt & 7) * 2;
#pragma unroll
        for (int r = NR; r < N; ++r)
          *reinterpret_cast<__nv_bfloat16*>(pb + r * 128 + ((ck ^ (r & 7)) << 4)) = __float2bfloat16_rn(0.f);
      }
    }
    int g = 0;
    bool ok = !s_abort;     // a failed wait is acted on only by a vote at the next stage
    // the next item with pages after `it` (for the Q one segment ahead)
    auto next_with_pages = [&](int it) {
      for (int k = it + 1; k < it1; ++k)
        if (draft_item(p, k).npg > 0) return k;
      return it1;
    };
    for (int it = it0; it < it1; ++it) {
      const DItem d = d0;                                  // the CTA's one item
      const size_t rowbase = (size_t)d.b * p.Hq + (size_t)d.h * p.G;
      const int slot_idx = d.u * p.parts + d.k;            // partial slot of a piece
      if (d.npg == 0) {
        // nothing to attend: an unusable length (first piece writes zeros and
        // lse -inf) or an empty piece of a split unit (an empty partial)
        if (d.bad) {
          if (d.k == 0) write_empty_unit<__nv_bfloat16>(p, d.b, d.h, tid, 128);
          continue;
        }
        if (p.parts == 1) continue;                        // cannot happen: a usable unit keeps >= 1 page
        for (int i = tid; i < p.rows * D; i += 128) p.part_o[(size_t)slot_idx * p.rows * D + i] = 0.f;
        if (tid < p.rows) {
          p.part_ml[((size_t)slot_idx * p.rows + tid) * 2] = -INFINITY;
          p.part_ml[((size_t)slot_idx * p.rows + tid) * 2 + 1] = 0.f;
        }
      } else {
        const int nxt = next_with_pages(it);
        const bool has_next = nxt < it1;
        if (has_next) {
          const DItem dn = draft_item(p, nxt);
          q_fetch(dn.b, dn.h);                             // lands while this item runs
        }
        const int nst = (d.npg + ppt - 1) / ppt;
        const int Lb = d.L;
        if (tid < N) s_nu[tid] = kNuInit;
        float l[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) l[r] = 0.f;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        bool abort_all = false;
        for (int j = 0; j < nst; ++j, ++g) {
          const int st = g % NS, sb = g & 1;
          ok &= mbar_wait(BAR(B_SFULL + sb), (g >> 1) & 1, &s_abort, p.status) &&
                mbar_wait(BAR(B_FULL + st), (g / NS) & 1, &s_abort, p.status);
          tc_fence_after();
          const int lp = s_stage_lp[st][tid >> log2P];
          const int pos = lp * p.P + (tid & (p.P - 1));
          const bool valid = lp >= 0 && pos < Lb;
          float s[NR];
          auto load_s = [&]() {
            tmem_ld_cols<NR>(tmem + lane_base + L::kColS + sb * N, s);
            tmem_wait_ld();
            if (!valid) {
#pragma unroll
              for (int r = 0; r < NR; ++r) s[r] = -INFINITY;
            }
          };
          load_s();
          float ymax = -INFINITY;
#pragma unroll
          for (int r = 0; r < NR; r += 4) {
            const float4 v = *reinterpret_cast<const float4*>(&s_nu[r]);
            ymax = fmaxf(fmaxf(ymax, fmaf(s[r], c, v.x)), fmaf(s[r + 1], c, v.y));
            ymax = fmaxf(fmaxf(ymax, fmaf(s[r + 2], c, v.z)), fmaf(s[r + 3], c, v.w));
          }
          const int cnt = wg_count(!ok || ymax > kTau);
          bool rescale_o = false;
          if (cnt > 0) {
            if (wg_count(!ok) > 0) { abort_all = true; break; }
            wg_rows_reduce<NR, true>(s, s_red, s_mx, q4, lane, tid);
            if (tid < NR) {
              const float m_old = -s_nu[tid];
              const float m_new = fmaxf(m_old, s_mx[tid] * c);
              s_alpha[tid] = ex2(m_old - m_new);
              s_nu[tid] = -m_new;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
            for (int r = 0; r < NR; r += 4) {
              const float4 a = *reinterpret_cast<const float4*>(&s_alpha[r]);
              l[r] *= a.x; l[r + 1] *= a.y; l[r + 2] *= a.z; l[r + 3] *= a.w;
            }
            load_s();
            rescale_o = j > 0;
          }
#pragma unroll
          for (int r = 0; r < NR; r += 4) {
            const float4 v = *reinterpret_cast<const float4*>(&s_nu[r]);
            s[r] = ex2(fmaf(s[r], c, v.x));
            s[r + 1] = ex2(fmaf(s[r + 1], c, v.y));
            s[r + 2] = ex2(fmaf(s[r + 2], c, v.z));
            s[r + 3] = ex2(fmaf(s[r + 3], c, v.w));
            l[r] += s[r]; l[r + 1] += s[r + 1]; l[r + 2] += s[r + 2]; l[r + 3] += s[r + 3];
          }
          const int gw = g - ((rescale_o || PB == 1) ? 1 : 2);
          if (gw >= 0) ok &= mbar_wait(BAR(B_ODONE + (gw & 1)), (gw >> 1) & 1, &s_abort, p.status);
          tc_fence_after();
          if (rescale_o) {
            float o[NR];
            tmem_ld_cols<NR>(tmem + lane_base + L::kColO, o);
            tmem_wait_ld();
#pragma unroll
            for (int r = 0; r < NR; ++r) o[r] *= s_alpha[r];
            tmem_st_cols<NR>(tmem + lane_base + L::kColO, o);
            tmem_wait_st();
          }
          {
            const int half = tid >> 6, tt = tid & 63;
            uint8_t* pb = sP + (g % PB) * L::kPBytes + half * (N * 128) + (tt & 7) * 2;
            const int ck = tt >> 3;
#pragma unroll
            for (int r = 0; r < NR; ++r)
              *reinterpret_cast<__nv_bfloat16*>(pb + r * 128 + ((ck ^ (r & 7)) << 4)) = __float2bfloat16_rn(s[r]);
          }
          if (!valid) {
            uint8_t* sV = sKV + st * 2 * L::kTileBytes + L::kTileBytes + tid * 128;
#pragma unroll
            for (int hh = 0; hh < L::kHalves; ++hh)
#pragma unroll
              for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(sV + hh * (kTok * 128) + k * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(BAR(B_PFULL + (g & 1)));
        }
        if (abort_all) break;                              // uniform: decided by wg_count
        if (has_next) q_store();                           // the item's last QK is done
        // ---- epilogue: row sums, then O^T / l
        wg_rows_reduce<NR, false>(l, s_red, s_alpha, q4, lane, tid);
        const bool single = p.parts == 1;
        if (tid < p.rows) {
          const float lt = s_alpha[tid], m = -s_nu[tid];
          if (single) {
            if (p.lse) p.lse[rowbase + tid] = lt > 0.f ? (m + log2f(lt)) * kLn2 : -INFINITY;
          } else {
            const size_t pi = (size_t)slot_idx * p.rows + tid;
            p.part_ml[pi * 2] = lt > 0.f ? m : -INFINITY;
            p.part_ml[pi * 2 + 1] = lt;
          }
          s_alpha[tid] = lt > 0.f ? 1.f / lt : 0.f;
        }
        ok &= mbar_wait(BAR(B_ODONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, &s_abort, p.status);
        tc_fence_after();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        {
          float o[NR];
          tmem_ld_cols<NR>(tmem + lane_base + L::kColO, o);
          tmem_wait_ld();
          if (d_mine >= 0) {
            if (single) {
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + rowbase * D + d_mine;
#pragma unroll
              for (int r = 0; r < NR; ++r)
                if (r < p.rows) dst[(size_t)r * D] = __float2bfloat16_rn(o[r] * s_alpha[r]);
            } else {
              float* dst = p.part_o + (size_t)slot_idx * p.rows * D + d_mine;
#pragma unroll
              for (int r = 0; r < NR; ++r)
                if (r < p.rows) dst[(size_t)r * D] = o[r];
            }
          }
        }
        tc_fence_before();
      }
      if (p.parts > 1 && !d.bad) {
        // pieces of a split unit: the last to finish merges them
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (tid == 0) s_ticket = atomicAdd(p.tickets + d.u, 1u);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (s_ticket == p.parts - 1) {
          __threadfence();
          combine_partials<__nv_bfloat16>(p, d.b, d.h, d.u * p.parts, p.parts, 128);
          if (tid == 0) p.tickets[d.u] = 0u;
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");    // s_alpha / s_nu reads done
    }
  }

  // ---- teardown: every role is done; wait for the MMAs, free TMEM
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kDfMma) {
    tc_fence_after();
    if (lane == 0) mbar_wait_drain(BAR(B_TD), 0, p.status);
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool draft_fused_supported(const s3r_paged_kv& kv, int32_t budget_pages) {
  const int G = kv.num_q_heads / kv.num_kv_heads;
  const long units = (long)kv.num_seqs * kv.num_kv_heads;
  int sms = device_sm_count();
  if (sms > kMaxPersistentCtas) sms = kMaxPersistentCtas;
  return kv.dtype == S3R_BF16 && G <= 8 && budget_pages >= 1 && budget_pages <= kDfMaxBudget &&
         kv.max_pages_per_seq <= kDfMaxPages && (kv.page_size == 16 || kv.page_size == 64) &&
         (kv.head_dim == 64 || kv.head_dim == 128) && units <= sms;
}

template <int D>
static cudaError_t prepare_d(const s3r_paged_kv& kv, int32_t budget_pages, DraftLaunch* dl) {
  dl->smem = DfLay<D>::kDynBytes + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(draft_fused_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dl->smem);
  if (e != cudaSuccess) return e;
  // the largest piece count (at most 4, at most the budget) whose clusters
  // are all resident at once: a second wave would double the time
  const int units = kv.num_seqs * kv.num_kv_heads;
  while (dl->parts > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * dl->parts);
    cfg.blockDim = dim3(kDfThreads);
    cfg.dynamicSmemBytes = dl->smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = dl->parts;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, draft_fused_kernel<D>, &cfg) == cudaSuccess && clusters >= units)
      break;
    (void)cudaGetLastError();
    dl->parts >>= 1;
  }
  dl->grid = units * dl->parts;
  return cudaSuccess;
}

cudaError_t prepare_draft_fused(const s3r_paged_kv& kv, int32_t budget_pages, DraftLaunch* dl) {
  if (!make_cache_map(&dl->mk, kv.k_cache, kv) || !make_cache_map(&dl->mv, kv.v_cache, kv))
    return cudaErrorInvalidValue;
  int sms = device_sm_count();
  if (sms > kMaxPersistentCtas) sms = kMaxPersistentCtas;
  const int units = kv.num_seqs * kv.num_kv_heads;
  int parts = sms / units;
  if (parts > 4) parts = 4;
  if (parts > budget_pages) parts = budget_pages;
  if (parts == 3) parts = 2;                           // cluster sizes 1, 2, 4
  if (parts < 1) parts = 1;
  dl->parts = parts;
  return kv.head_dim == 64 ? prepare_d<64>(kv, budget_pages, dl) : prepare_d<128>(kv, budget_pages, dl);
}

cudaError_t launch_draft_fused(const s3r_paged_kv& kv, const DraftLaunch& dl, const AttnParams& p, cudaStream_t st) {
  if (kv.head_dim == 64)
    return launch_kernel(draft_fused_kernel<64>, dim3(dl.grid), dim3(kDfThreads), dl.smem, st, dl.parts, dl.mk,
                         dl.mv, p);
  return launch_kernel(draft_fused_kernel<128>, dim3(dl.grid), dim3(kDfThreads), dl.smem, st, dl.parts, dl.mk,
                       dl.mv, p);
}

}  // namespace s3r
