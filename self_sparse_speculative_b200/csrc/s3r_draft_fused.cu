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
// kernel (persistent CTAs claiming units from a workspace counter) and the
// split-KV attention kernel instead.
//
// Selection of a unit (all 256 threads of the CTA):
//   score(p) = sum_g sum_d max(q_g,d kmin_p,d, q_g,d kmax_p,d) for p < n_b,
//   folded per channel into A max(kmin, kmax) + B min(kmin, kmax) with
//   A = sum_g max(q_g, 0) and B = sum_g min(q_g, 0) (exact in real arithmetic),
//   and the tail page n_b - 1 is summarised from K itself (its keys change
//   while the sequence decodes). The summary rows are read from global memory
//   (a unit's rows are 2 D bytes per page, too small for bulk copies to pay);
//   the tail page's K is bulk-copied into the K/V ring, which is still empty,
//   while the other pages are scored. Scores are accumulated in float32
//   (packed bf16x2 max / min, f32x2 multiply-adds) with one rigorous bound E
//   on the rounding error of every score of the unit; warp bitonic sorts and a
//   merge tree keeping the top 32 or 64 (a radix select past that) find the
//   budget-th largest float32 score s_B. A page with s_p > s_B + 2E is kept
//   for certain, one with s_p < s_B - 2E dropped; the pages in between are
//   re-scored in float64 and ranked (ties to the lower page) only when they
//   outnumber the places left, so the kept set is the float64 top-B. It goes,
//   in ascending page order, into a list in shared memory.
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
  static constexpr uint32_t kTailBytes = 64 * D * 2;               // K of one page (P <= 64)
  static constexpr uint32_t kOffKeys = T::kOffKV + kRing;          // u64 [kDfMaxPages]
  static constexpr uint32_t kOffPhys = kOffKeys + 8 * kDfMaxPages; // int [kDfMaxPages]
  static constexpr uint32_t kOffList = kOffPhys + 4 * kDfMaxPages; // int2 [kDfMaxBudget]
  static constexpr uint32_t kOffAB = kOffList + 8 * kDfMaxBudget;  // double [2][D]
  static constexpr uint32_t kOffTail = kOffAB + 2 * 8 * D;         // bf16 [2][D]
  static constexpr uint32_t kOffHist = kOffTail + 2 * 2 * D;       // u32 [256]
  static constexpr uint32_t kDynBytes = kOffHist + 4 * 256;
  static_assert(4 * kDfMaxPages >= kDfThreads * 16, "tail scratch fits in the key array's upper half");
  static_assert(kTailBytes + 12 * kDfMaxPages <= kRing, "tail rows and band scratch fit in the ring");
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
  float wmax[8];
  float emax[4];               // per cluster rank: the largest summary magnitude |kmin|, |kmax|
  uint32_t digit, want;
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
// and the folded query weights of its KV head. The whole block-table row and
// the query are loaded whatever the length, so these loads do not wait for
// the context length's (entries past the last page are never used).
template <int D>
__device__ void sel_prepare(const AttnParams& p, const DItem& d, int tg, int nthr, const SelSmem& sm) {
  const int32_t* bt = p.block_table + (size_t)d.b * p.max_pages;
  for (int i = tg; i < p.max_pages; i += nthr) sm.phys[i] = __ldg(bt + i);
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

// Order-preserving 32-bit image of a float score, and back.
__device__ __forceinline__ uint32_t order_key32(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u >> 31) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key32_value(uint32_t k) {
  return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k);
}

// Packed helpers: max / min of two bf16 pairs (exact), the pair as two
// floats (exact), and two independent fused multiply-adds (each rounded once).
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ unsigned long long bf2_pair(uint32_t u) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(u << 16), "r"(u & 0xFFFF0000u));
  return d;
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_pair(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float f2_sum(unsigned long long v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}

// Rounding bound of the float32 scores (u = 2^-24). A product A_c x_c meets
// one rounding of A_c to float32, at most D/64 in its lane's multiply-add
// chain (channel pairs: even and odd channels accumulate apart), two where
// the lane's four chains are added and five in the warp's reduction: at most
// 10 at D = 128 (9 at D = 64), the tail page's score at most 11. A sum
// evaluated so is within gamma_11 = 11 u / (1 - 11 u) of the exact value
// times the sum of the terms' magnitudes (N. Higham, Accuracy and Stability
// of Numerical Algorithms, 2002, section 3.1), and that sum is at most
// W M with W = sum_c (A_c + |B_c|) and M the largest |kmin|, |kmax| of the
// unit's pages; 16 u W M covers it (and the roundings of the product).
constexpr double kScoreGamma = 16.0 * 5.9604644775390625e-8;

// Float32 scores of pages [g0, g1) (none of them the tail page) of KV head
// h into the 32-bit keys, the summary rows read from global memory (a unit's
// 2 D bytes of a page are not contiguous with the next page's, so they come
// as many small pieces; plain loads keep 2 kU of them in flight per lane).
// kU pages (16 or 8) per warp and round, each lane holding D / 32 channels
// of every page as bf16 pairs: max / min per pair, then packed multiply-adds;
// the kU page sums are reduced across the warp together (halving exchanges:
// lane l ends with page l % kU). Returns the largest |kmin|, |kmax| the
// thread saw (0 if none), for the rounding bound.
template <int D, int kU>
__device__ float score_pages(const AttnParams& p, int h, int g0, int g1, int tg, int nthr, const SelSmem& sm,
                             uint32_t* keys32) {
  constexpr int CPL = D / 32, PPL = CPL / 2;              // channels and channel pairs per lane
  using Raw = typename std::conditional<CPL == 4, uint2, uint32_t>::type;
  const int lane = tg & 31, gw = tg >> 5, nw = nthr >> 5;
  unsigned long long wa[PPL], wb[PPL];
#pragma unroll
  for (int c = 0; c < PPL; ++c) {
    const int ch = lane * CPL + 2 * c;
    wa[c] = f2_pair(static_cast<float>(sm.ab[ch]), static_cast<float>(sm.ab[ch + 1]));
    wb[c] = f2_pair(static_cast<float>(sm.ab[D + ch]), static_cast<float>(sm.ab[D + ch + 1]));
  }
  uint32_t rmax = 0xFF80FF80u, rmin = 0x7F807F80u;         // bf16 pairs (-inf, -inf), (+inf, +inf)
  for (int pg0 = g0 + gw * kU; pg0 < g1; pg0 += nw * kU) {
    Raw lo[kU], hi[kU];
    bool ok[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int pg = pg0 + u;
      const int ph = pg < g1 ? sm.phys[pg] : -1;
      ok[u] = ph >= 0 && ph < p.num_pages_total;
      const size_t base = ((size_t)ph * p.Hkv + h) * D;
      if (ok[u]) {
        lo[u] = __ldg(reinterpret_cast<const Raw*>(static_cast<const __nv_bfloat16*>(p.kmin) + base) + lane);
        hi[u] = __ldg(reinterpret_cast<const Raw*>(static_cast<const __nv_bfloat16*>(p.kmax) + base) + lane);
      }
    }
    float acc[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      unsigned long long sx = 0ull, sn = 0ull;            // (+0, +0)
      if (ok[u]) {
        uint32_t lw[PPL], hw[PPL];
        if constexpr (CPL == 4) { lw[0] = ((uint2&)lo[u]).x; lw[1] = ((uint2&)lo[u]).y; hw[0] = ((uint2&)hi[u]).x; hw[1] = ((uint2&)hi[u]).y; }
        else { lw[0] = (uint32_t&)lo[u]; hw[0] = (uint32_t&)hi[u]; }
#pragma unroll
        for (int w = 0; w < PPL; ++w) {
          const uint32_t x = bmax2(lw[w], hw[w]), n = bmin2(lw[w], hw[w]);
          rmax = bmax2(rmax, x);
          rmin = bmin2(rmin, n);
          sx = ffma2(wa[w], bf2_pair(x), sx);
          sn = ffma2(wb[w], bf2_pair(n), sn);
        }
      }
      acc[u] = f2_sum(sx) + f2_sum(sn);
    }
#pragma unroll
    for (int w = kU / 2; w >= 1; w >>= 1) {
      const bool up = (lane & w) != 0;
#pragma unroll
      for (int k = 0; k < w; ++k) {
        const float send = up ? acc[k] : acc[k + w];
        const float keep = up ? acc[k + w] : acc[k];
        acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, w);
      }
    }
    // lane l now holds page l % kU summed over its kU-lane group; the groups
    // combine (five additions on every path whatever kU)
    float v = acc[0];
#pragma unroll
    for (int o = kU; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int pg = pg0 + (lane & (kU - 1));
    if (lane < kU && pg < g1) {
      bool okp = false;
#pragma unroll
      for (int u = 0; u < kU; ++u) okp = (u == lane) ? ok[u] : okp;
      if (!okp) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      keys32[pg] = okp ? order_key32(v) : 0u;
    }
  }
  // the largest magnitude: max over channels of max(x, -n) (every |kmin|,
  // |kmax| is at most that); NaN summaries are passed over as by the maxima
  float xa, xb, na, nb;
  bf2(rmax, xa, xb);
  bf2(rmin, na, nb);
  return fmaxf(0.f, fmaxf(fmaxf(xa, xb), -fminf(na, nb)));
}

// Bitonic network over the 32 lanes: descending order (lane 0 the largest).
// A lane pair (i, i ^ j) keeps the larger value at the lower lane within a
// descending run of length k.
__device__ __forceinline__ uint32_t warp_sort_desc(uint32_t v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool desc = (lane & k) == 0 || k == 32;
      const bool lower = (lane & j) == 0;
      v = (lower == desc) ? max(v, o) : min(v, o);
    }
  return v;
}
// The 32 largest of two descending 32-lists, descending: the lane-wise
// maximum of one list and the other reversed is bitonic and holds them;
// a half-cleaner cascade sorts it.
__device__ __forceinline__ uint32_t warp_merge_top(uint32_t a, uint32_t b_rev, int lane) {
  uint32_t v = max(a, b_rev);
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint32_t o = __shfl_xor_sync(0xffffffffu, v, j);
    v = ((lane & j) == 0) ? max(v, o) : min(v, o);
  }
  return v;
}
// The B-th largest (B <= 32) of keys[0..n) by the 256 threads: each warp
// sorts 32 keys at a time and keeps the top 32 of what it has seen (keys
// tg, tg + 256, ...), then a tree of merges across the warps keeps the top 32.
__device__ uint32_t top32_kth(const uint32_t* keys, int n, int B, int tg, int barid, uint32_t* xch) {
  const int lane = tg & 31, gw = tg >> 5;
  uint32_t v = warp_sort_desc(tg < n ? keys[tg] : 0u, lane);
  for (int base = kDfThreads; base < n; base += kDfThreads) {        // uniform: n is
    const int i = base + tg;
    const uint32_t w = warp_sort_desc(i < n ? keys[i] : 0u, lane);
    v = warp_merge_top(v, __shfl_sync(0xffffffffu, w, 31 - lane), lane);
  }
#pragma unroll
  for (int step = 1; step < 8; step <<= 1) {
    if ((gw & (2 * step - 1)) == step) xch[(gw - step) * 32 + 31 - lane] = v;   // reversed, for the partner
    grp_sync(barid, kDfThreads);
    if ((gw & (2 * step - 1)) == 0) v = warp_merge_top(v, xch[gw * 32 + lane], lane);
    grp_sync(barid, kDfThreads);
  }
  if (gw == 0 && lane == B - 1) xch[0] = v;
  grp_sync(barid, kDfThreads);
  const uint32_t k = xch[0];
  grp_sync(barid, kDfThreads);
  return k;
}

// Descending 64-lists held by a warp as two registers: element e is lane
// e % 32 of register e / 32 (x0 the larger half). half_clean32 sorts a
// bitonic 32-list (one register) descending.
__device__ __forceinline__ uint32_t half_clean32(uint32_t v, int lane) {
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint32_t o = __shfl_xor_sync(0xffffffffu, v, j);
    v = ((lane & j) == 0) ? max(v, o) : min(v, o);
  }
  return v;
}
// 64 keys (a, b: one per lane each) sorted descending into (x0, x1): two
// sorted halves, then the bitonic merge of one with the other reversed.
__device__ __forceinline__ void warp_sort64_desc(uint32_t a, uint32_t b, int lane, uint32_t& x0, uint32_t& x1) {
  const uint32_t sa = warp_sort_desc(a, lane);
  const uint32_t sb = __shfl_sync(0xffffffffu, warp_sort_desc(b, lane), 31 - lane);
  x0 = half_clean32(max(sa, sb), lane);
  x1 = half_clean32(min(sa, sb), lane);
}
// The 64 largest of descending 64-lists X and Y, descending: element e of
// max(X, Y reversed) is bitonic and holds them (Y reversed: element e is
// Y[63 - e]); a distance-32 step in the lane, then each half cleaned.
__device__ __forceinline__ void warp_merge_top64(uint32_t& x0, uint32_t& x1, uint32_t y0, uint32_t y1, int lane) {
  const uint32_t z0 = max(x0, __shfl_sync(0xffffffffu, y1, 31 - lane));
  const uint32_t z1 = max(x1, __shfl_sync(0xffffffffu, y0, 31 - lane));
  x0 = half_clean32(max(z0, z1), lane);
  x1 = half_clean32(min(z0, z1), lane);
}
// The B-th largest (32 < B <= 64) of keys[0..n) by the 256 threads: each
// warp sorts 64 keys at a time and keeps the top 64 of what it has seen, then
// a tree of merges across the warps keeps the top 64. xch: 2 KB.
__device__ uint32_t top64_kth(const uint32_t* keys, int n, int B, int tg, int barid, uint32_t* xch) {
  const int lane = tg & 31, gw = tg >> 5;
  uint32_t x0 = 0u, x1 = 0u;
  for (int base = 0; base < n; base += 2 * kDfThreads) {           // uniform: n is
    const int i = base + gw * 64 + lane;
    uint32_t y0, y1;
    warp_sort64_desc(i < n ? keys[i] : 0u, i + 32 < n ? keys[i + 32] : 0u, lane, y0, y1);
    if (base == 0) { x0 = y0; x1 = y1; }
    else warp_merge_top64(x0, x1, y0, y1, lane);
  }
#pragma unroll
  for (int step = 1; step < 8; step <<= 1) {
    if ((gw & (2 * step - 1)) == step) {
      xch[(gw - step) * 64 + lane] = x0;
      xch[(gw - step) * 64 + 32 + lane] = x1;
    }
    grp_sync(barid, kDfThreads);
    if ((gw & (2 * step - 1)) == 0) warp_merge_top64(x0, x1, xch[gw * 64 + lane], xch[gw * 64 + 32 + lane], lane);
    grp_sync(barid, kDfThreads);
  }
  if (gw == 0 && lane == ((B - 1) & 31)) xch[0] = (B - 1) < 32 ? x0 : x1;
  grp_sync(barid, kDfThreads);
  const uint32_t k = xch[0];
  grp_sync(barid, kDfThreads);
  return k;
}

// Rank of 32-bit key kp (page i) among keys[0..n): the keys above it plus
// the equal keys of lower pages. keys 16-byte aligned; four keys per load.
__device__ __forceinline__ int rank32(const uint32_t* keys, int n, uint32_t kp, int i) {
  int r0 = 0, r1 = 0;
  int j = 0;
  const uint4* k4 = reinterpret_cast<const uint4*>(keys);
  for (; j + 4 <= n; j += 4) {
    const uint4 a = k4[j >> 2];
    r0 += (a.x > kp) + (a.x == kp && j < i) + (a.y > kp) + (a.y == kp && j + 1 < i);
    r1 += (a.z > kp) + (a.z == kp && j + 2 < i) + (a.w > kp) + (a.w == kp && j + 3 < i);
  }
  for (; j < n; ++j) r0 += (keys[j] > kp) + (keys[j] == kp && j < i);
  return r0 + r1;
}

// The want-th largest (1-based) of keys[0..n), want <= n: 8-bit digits from
// the top; per digit a shared-memory histogram of the keys that still match
// the prefix (one atomic per distinct digit and warp), and warp 0 finds the
// digit whose bin holds the want-th key. All threads of the group.
__device__ uint32_t radix_kth_largest(const uint32_t* keys, int n, int want, int tg, int nthr, int barid,
                                      unsigned* hist, SelScratch& sc) {
  const int lane = tg & 31, gw = tg >> 5;
  uint32_t prefix = 0, mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tg; i < 256; i += nthr) hist[i] = 0u;
    grp_sync(barid, nthr);
    for (int i0 = 0; i0 < n; i0 += nthr) {
      const int i = i0 + tg;
      const uint32_t k = i < n ? keys[i] : 0u;
      const bool act = i < n && (k & mask) == prefix;
      const uint32_t dig = act ? (k >> shift) & 255u : 0x100u | (uint32_t)lane;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (unsigned)__popc(peers));
    }
    grp_sync(barid, nthr);
    if (gw == 0) {
      // lane l holds bins 255 - 8 l .. 248 - 8 l (from the top)
      unsigned cnt[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cnt[j] = hist[255 - (lane * 8 + j)]; tot += cnt[j]; }
      unsigned inc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned exc = inc - tot;
      const unsigned w = (unsigned)want;
      if (exc < w && w <= inc) {
        unsigned c = exc;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (c + cnt[j] >= w && c < w) { sc.digit = 255u - (unsigned)(lane * 8 + j); sc.want = w - c; }
          c += cnt[j];
        }
      }
    }
    grp_sync(barid, nthr);
    prefix |= sc.digit << shift;
    mask |= 255u << shift;
    want = (int)sc.want;
    grp_sync(barid, nthr);                             // sc is rewritten by the next digit
  }
  return prefix;
}

// Float64 score of page pg of the unit (warp-wide; every lane gets it): the
// summaries from global memory, the tail page from sm.tail.
template <int D>
__device__ double score_page64(const AttnParams& p, const DItem& d, int pg, const SelSmem& sm, int lane) {
  constexpr int CPL = D / 32;
  const int ph = sm.phys[pg];
  double a0 = 0.0, a1 = 0.0;
  if (ph >= 0 && ph < p.num_pages_total) {
    const bool tail = pg == d.n_b - 1;
    const __nv_bfloat16* mn = static_cast<const __nv_bfloat16*>(p.kmin) + ((size_t)ph * p.Hkv + d.h) * D;
    const __nv_bfloat16* mx = static_cast<const __nv_bfloat16*>(p.kmax) + ((size_t)ph * p.Hkv + d.h) * D;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int ch = lane * CPL + c;
      const float l = tail ? __bfloat162float(sm.tail[ch]) : __bfloat162float(mn[ch]);
      const float r = tail ? __bfloat162float(sm.tail[D + ch]) : __bfloat162float(mx[ch]);
      a0 = fma(sm.ab[ch], static_cast<double>(fmaxf(l, r)), a0);
      a1 = fma(sm.ab[D + ch], static_cast<double>(fminf(l, r)), a1);
    }
  }
  double v = a0 + a1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
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

// The kept pages of item d's unit, ascending, into `list` (logical,
// physical). All threads of the CTA, after sel_prepare. It reads only inputs
// (summaries, the tail page's keys) and writes only shared memory (and the
// status word), so it runs before the grid-dependency wait.
// clustered: the unit is shared by the p.parts CTAs of this cluster (rank =
// d.k); each scores its share of the pages and sends its keys and its bound
// to the first CTA, which selects and hands the list back.
// KU: pages per warp and scoring round (registers: two summary pieces each).
template <int D, int KU = 16>
__device__ void select_unit(const AttnParams& p, const DItem& d, int2* list, const SelSmem& sm, SelScratch& sc,
                            uint8_t* stage, uint32_t bar_g0, uint32_t* g0_phase, bool clustered, volatile int* abort) {
  using Lay = DfLay<D>;
  constexpr int nthr = kDfThreads, barid = kBarAll;
  const int tg = threadIdx.x, lane = tg & 31, gw = tg >> 5;
  for (int k = tg; k < p.budget; k += nthr) list[k] = make_int2(-1, -1);
  if (d.bad) {
    if (d.k == 0 && tg == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
    return;
  }
  const int n_b = d.n_b;
  if (n_b <= p.budget) {
    for (int k = tg; k < n_b; k += nthr) list[k] = make_int2(k, sm.phys[k]);
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
  uint32_t* keys32 = reinterpret_cast<uint32_t*>(sm.keys);   // [kDfMaxPages], the array's lower half
  float4* scratch = reinterpret_cast<float4*>(sm.keys + kDfMaxPages / 2);   // its upper half
  bool ok = true;
  float mmax = 0.f;                                      // the largest summary magnitude seen
  // the tail page's K (when in the share) bulk-copied into the empty ring
  // while the other pages are scored from their summaries
  if (has_tail && tail_ok && tg == 0) {
    const uint32_t bytes = (uint32_t)valid * D * 2;
    mbar_arrive_expect_tx(bar_g0, bytes);
    bulk_load(smem_addr(stage), tail_src, bytes, bar_g0);
  }
  const int e = min(s1, tail);                           // the share's pages other than the tail
  mmax = score_pages<D, KU>(p, d.h, s0, e, tg, nthr, sm, keys32);
  if (has_tail && tail_ok) {
    ok = grp_all(mbar_wait(bar_g0, *g0_phase, abort, p.status), barid, nthr);
    *g0_phase ^= 1u;
    if (ok) {
      tail_minmax<D>(reinterpret_cast<const __nv_bfloat16*>(stage), valid, tg, nthr, barid, sm, scratch);
    }
    fence_proxy_async_smem();                            // reads of the staged rows before copies reuse them
    grp_sync(barid, nthr);
  }
  // the tail page, scored from its fresh min / max (first warp)
  if (ok && has_tail && gw == 0) {
    constexpr int CPL = D / 32;
    float a0 = 0.f, a1 = 0.f;
    if (tail_ok) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int ch = lane * CPL + c;
        const float l = __bfloat162float(sm.tail[ch]), r = __bfloat162float(sm.tail[D + ch]);
        const float wa = static_cast<float>(sm.ab[ch]), wb = static_cast<float>(sm.ab[D + ch]);
        a0 = fmaf(wa, fmaxf(l, r), a0);
        a1 = fmaf(wb, fminf(l, r), a1);
        mmax = fmaxf(mmax, fmaxf(fabsf(l), fabsf(r)));
      }
    }
    float v = a0 + a1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      if (!tail_ok) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      keys32[tail] = tail_ok ? order_key32(v) : 0u;
    }
  }
  // the CTA's largest summary magnitude
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  if (lane == 0) sc.wmax[gw] = mmax;
  grp_sync(barid, nthr);
  if (tg == 0) {
    float m = 0.f;
    for (int w = 0; w < nthr / 32; ++w) m = fmaxf(m, sc.wmax[w]);
    sc.emax[rank] = m;
  }
  grp_sync(barid, nthr);
  if (clustered) {
    // every share's keys and bound into the first CTA
    cluster_sync_all();                                  // every CTA has scored
    if (rank != 0) {
      for (int pg = s0 + tg; pg < s1; pg += nthr) st_cluster_u32(&keys32[pg], 0u, keys32[pg]);
      if (tg == 0) st_cluster_u32(&sc.emax[rank], 0u, __float_as_uint(sc.emax[rank]));
      if (has_tail) {
        // the tail page's fresh min / max, for a float64 re-score there
        const uint32_t* t32 = reinterpret_cast<const uint32_t*>(sm.tail);
        for (int i = tg; i < D; i += nthr) st_cluster_u32(&t32[i], 0u, t32[i]);
      }
    }
    cluster_sync_all();                                  // the first CTA holds every key
  }
  ok = grp_all(ok, barid, nthr);
  if (rank == 0 && ok) {
    const int B = p.budget;
    // the bound: 16 u W M (W = sum_c A_c + |B_c|, exact in float64; M the
    // largest magnitude over every share), rounded up to float32
    float M = 0.f;
    for (int r = 0; r < parts; ++r) M = fmaxf(M, sc.emax[r]);
    double W = 0.0;
    for (int c = lane; c < D; c += 32) W += sm.ab[c] - sm.ab[D + c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
    const float E = __double2float_ru(kScoreGamma * W * static_cast<double>(M));
    // the B-th largest float32 score, and the band in which float32 cannot
    // order pages: |s_p - s_B| <= 2E
    uint32_t kB;
    if (B <= 32) {
      kB = top32_kth(keys32, n_b, B, tg, barid, reinterpret_cast<uint32_t*>(stage));   // the ring is idle
    } else if (B <= 64) {
      kB = top64_kth(keys32, n_b, B, tg, barid, reinterpret_cast<uint32_t*>(stage));
    } else if (n_b <= nthr) {
      // one key per thread: its rank among all (ties to the lower page)
      if (tg < n_b && rank32(keys32, n_b, keys32[tg], tg) == B - 1) sc.digit = keys32[tg];
      grp_sync(barid, nthr);
      kB = sc.digit;
      grp_sync(barid, nthr);
    } else {
      kB = radix_kth_largest(keys32, n_b, B, tg, nthr, barid, sm.hist, sc);
    }
    // the band's edges as keys: a float score s has s > hi iff s > RD(hi)
    // and s >= lo iff s >= RU(lo) (float32 roundings of the float64 edges);
    // a zero edge takes the key of the zero that makes both zeros compare as
    // floats do; keys above +inf's are NaN scores (neither kept nor in band)
    const double sB = static_cast<double>(key32_value(kB));
    const double hiB = sB + 2.0 * static_cast<double>(E), loB = sB - 2.0 * static_cast<double>(E);
    const float hiF = __double2float_rd(hiB), loF = __double2float_ru(loB);
    const uint32_t kHi = order_key32(hiF == 0.f ? 0.f : hiF), kLo = order_key32(loF == 0.f ? -0.f : loF);
    constexpr uint32_t kInf = 0xFF800000u;               // order_key32(+inf)
    // each thread owns a run of consecutive pages (the list keeps page order);
    // the pages above the band and those in it, counted together
    const int per = (n_b + nthr - 1) / nthr;
    const int q0 = min(n_b, tg * per), q1 = min(n_b, q0 + per);
    int n_cnt = 0;
    for (int pg = q0; pg < q1; ++pg) {
      const uint32_t k = keys32[pg];
      n_cnt += (k <= kInf && k > kHi) ? 0x10000 : ((k <= kInf && k >= kLo) ? 1 : 0);
    }
    int tot;
    const int before = grp_exclusive_scan(n_cnt, tg, nthr, barid, sc, &tot);
    const int tot_in = tot >> 16, tot_unc = tot & 0xffff;
    const int need = B - tot_in;                         // places left for the band's pages
    if (tot_unc <= need) {
      // the whole band is kept (the common case): positions from the scan
      int pos = (before >> 16) + (before & 0xffff);
      for (int pg = q0; pg < q1; ++pg) {
        const uint32_t k = keys32[pg];
        if (k <= kInf && k >= kLo) {
          if (pos < B) list[pos] = make_int2(pg, sm.phys[pg]);
          ++pos;
        }
      }
    } else {
      // float64 scores of the band's pages, ranked among themselves (ties to
      // the lower page); the ring is idle until the list is done. Keep flags
      // one bit per page (the histogram's words).
      unsigned* keepbits = sm.hist;
      for (int i = tg; i < 256; i += nthr) keepbits[i] = 0u;
      unsigned long long* ukey = reinterpret_cast<unsigned long long*>(stage);           // [kDfMaxPages]
      int* upage = reinterpret_cast<int*>(stage + 8 * kDfMaxPages);                     // [kDfMaxPages]
      int j = before & 0xffff;
      for (int pg = q0; pg < q1; ++pg) {
        const uint32_t k = keys32[pg];
        if (k <= kInf && k >= kLo && k <= kHi) upage[j++] = pg;
      }
      grp_sync(barid, nthr);
      for (int u = gw; u < tot_unc; u += nthr / 32) {
        const double v = score_page64<D>(p, d, upage[u], sm, lane);
        if (lane == 0) ukey[u] = order_key(v);
      }
      grp_sync(barid, nthr);
      for (int u = tg; u < tot_unc; u += nthr)
        if (key_rank(ukey, tot_unc, ukey[u], u) < need) atomicOr(&keepbits[upage[u] >> 5], 1u << (upage[u] & 31));
      grp_sync(barid, nthr);
      // the list: pages above the band and the band's kept ones, in page order
      int n_keep = 0;
      for (int pg = q0; pg < q1; ++pg) {
        const uint32_t k = keys32[pg];
        n_keep += k <= kInf && (k > kHi || (k >= kLo && ((keepbits[pg >> 5] >> (pg & 31)) & 1u)));
      }
      int tot_keep;
      int pos = grp_exclusive_scan(n_keep, tg, nthr, barid, sc, &tot_keep);
      for (int pg = q0; pg < q1; ++pg) {
        const uint32_t k = keys32[pg];
        if (k <= kInf && (k > kHi || (k >= kLo && ((keepbits[pg >> 5] >> (pg & 31)) & 1u)))) {
          if (pos < B) list[pos] = make_int2(pg, sm.phys[pg]);
          ++pos;
        }
      }
    }
    fence_proxy_async_smem();                            // scratch in the ring before the copies reuse it
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
  __shared__ __align__(8) uint64_t s_bar[2 * NS + 9];
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
            B_QFULL = 2 * NS + 6, B_TD = 2 * NS + 7, B_G0 = 2 * NS + 8;
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
  // the selection and the first ring stages read only inputs, so they run
  // before the grid-dependency wait; every role takes the wait before it
  // touches an output or the workspace (the producer after its first NS
  // stages)
  uint32_t g0_phase = 0;
  select_unit<D>(p, d0, s_list, sm, s_sc, sKV, BAR(B_G0), &g0_phase, clustered, &s_abort);
  __syncthreads();

  if (warp == kDfProducer) {
    // ======================================================= producer warp
    const uint64_t pol = l2_policy_evict_first();
    int g = 0;
    bool waited = false;
    bool ok = __all_sync(0xffffffffu, !s_abort);
    for (int it = it0; it < it1 && ok; ++it) {
      const DItem d = d0;                                  // the CTA's one item
      const int2* list = s_list;
      const int nst = (d.npg + ppt - 1) / ppt;
      for (int j = 0; j < nst; ++j, ++g) {
        const int st = g % NS;
        if (g == NS && !waited) {                          // the ring's first fill went out before it
          pdl_wait();
          waited = true;
        }
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
    if (!waited) pdl_wait();
    if (lane == 0)
      for (int k = max(0, g - NS); k < g; ++k) mbar_wait_drain(BAR(B_FULL + k % NS), (k / NS) & 1, p.status);
  } else if (warp == kDfMma) {
    // ======================================================= MMA issuer
    pdl_wait();
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
    pdl_wait();
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
  } else {
    // ================================== selection helpers: the kept pages
    pdl_wait();
    if (d0.k == 0) {
      int32_t* out = p.selected_out + ((size_t)d0.b * p.Hkv + d0.h) * p.budget;
      for (int k = tid - 6 * 32; k < p.budget; k += kDfThreads - 6 * 32) out[k] = s_list[k].x;
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

// Page selection alone, for launches with more (sequence, KV head) units
// than SMs: persistent CTAs run the fused kernel's selection one unit after
// another, then write the kept pages' logical ids to selected_out and their
// physical ids to `phys_out` ([S, Hkv, budget], in the workspace) for the
// split-KV attention kernel. Small shared memory, so several CTAs share an
// SM and their summary loads overlap. Units are taken longest sequence first
// (every CTA ranks the context lengths, ties to the lower sequence, when
// there are at most kSelOrderMax sequences of unequal lengths), so the last
// claims are short units: CTA c takes position c first (scored before the
// grid-dependency wait), then claims positions from the workspace counter
// work[0] (after the wait: the previous call's selection resets it as it
// ends); the last CTA to finish (work[1]) returns both counters to zero.
template <int D>
struct SelOnlyLay {
  // the tail page's K, then the band scratch (float64 keys and pages)
  static constexpr uint32_t kStage =
      DfLay<D>::kTailBytes > 12u * kDfMaxPages ? DfLay<D>::kTailBytes : 12u * kDfMaxPages;
  static constexpr uint32_t kOffKeys = kStage;                      // u64 [kDfMaxPages]
  static constexpr uint32_t kOffPhys = kOffKeys + 8 * kDfMaxPages;  // int [kDfMaxPages]
  static constexpr uint32_t kOffList = kOffPhys + 4 * kDfMaxPages;  // int2 [kDfMaxBudget]
  static constexpr uint32_t kOffAB = kOffList + 8 * kDfMaxBudget;   // double [2][D]
  static constexpr uint32_t kOffTail = kOffAB + 2 * 8 * D;          // bf16 [2][D]
  static constexpr uint32_t kOffHist = kOffTail + 2 * 2 * D;        // u32 [256]
  static constexpr uint32_t kDynBytes = kOffHist + 4 * 256;
  static_assert(kStage >= 12 * kDfMaxPages, "band scratch fits in the tail stage");
};
constexpr int kSelOnlyCtasPerSm = 3;
constexpr int kSelOrderMax = 256;

template <int D>
__global__ void __launch_bounds__(kDfThreads, kSelOnlyCtasPerSm)
    select_only_kernel(const AttnParams p, int32_t* phys_out, uint32_t* work) {
  using Lay = SelOnlyLay<D>;
  extern __shared__ __align__(1024) uint8_t dyn_raw[];
  uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t s_bar[1];
  __shared__ int s_abort;
  __shared__ int s_unit;
  __shared__ SelScratch s_sc;
  __shared__ int s_len[kSelOrderMax];
  __shared__ int s_order[kSelOrderMax];                   // sequences, longest first
  const int tid = threadIdx.x;
  SelSmem sm;
  sm.keys = reinterpret_cast<unsigned long long*>(dyn + Lay::kOffKeys);
  sm.phys = reinterpret_cast<int*>(dyn + Lay::kOffPhys);
  sm.ab = reinterpret_cast<double*>(dyn + Lay::kOffAB);
  sm.tail = reinterpret_cast<__nv_bfloat16*>(dyn + Lay::kOffTail);
  sm.hist = reinterpret_cast<unsigned*>(dyn + Lay::kOffHist);
  int2* s_list = reinterpret_cast<int2*>(dyn + Lay::kOffList);
  if (tid == 0) {
    mbar_init(smem_addr(&s_bar[0]), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  const int units = p.S * p.Hkv;
  bool lpt = p.S <= kSelOrderMax;
  if (lpt) {
    int differs = 0;
    for (int b = tid; b < p.S; b += kDfThreads) {
      s_len[b] = __ldg(p.context_lens + b);
      differs |= s_len[b] != __ldg(p.context_lens);
    }
    lpt = __syncthreads_or(differs) != 0;                  // equal lengths: index order is as good
  }
  if (lpt) {
    for (int b = tid; b < p.S; b += kDfThreads) {
      const int L = s_len[b];
      int r = 0;
      for (int c = 0; c < p.S; ++c) r += s_len[c] > L || (s_len[c] == L && c < b);
      s_order[r] = b;
    }
    __syncthreads();
  }
  auto unit_at = [&](int k) {                              // claim position -> unit
    if (!lpt) return k;
    const int i = k / p.Hkv;
    return s_order[i] * p.Hkv + (k - i * p.Hkv);
  };
  uint32_t g0_phase = 0;
  bool waited = false;
  for (int k = blockIdx.x; k < units;) {
    const DItem d = draft_item(p, unit_at(k));             // p.parts == 1: item = unit
    sel_prepare<D>(p, d, tid, kDfThreads, sm);
    __syncthreads();
    select_unit<D, 8>(p, d, s_list, sm, s_sc, dyn, smem_addr(&s_bar[0]), &g0_phase, false, &s_abort);
    __syncthreads();
    if (!waited) {
      pdl_wait();                                          // outputs and the workspace from here on
      waited = true;
    }
    const size_t o = ((size_t)d.b * p.Hkv + d.h) * p.budget;
    for (int k = tid; k < p.budget; k += kDfThreads) {
      const int2 e = s_list[k];
      p.selected_out[o + k] = e.x;
      phys_out[o + k] = e.y;
    }
    // after a timed-out wait the tail stage may still be filling: claim no more
    if (tid == 0) s_unit = s_abort ? units : (int)(gridDim.x + atomicAdd(work, 1u));
    __syncthreads();                                       // s_unit; s_list and the stage are free again
    k = s_unit;
  }
  if (!waited) pdl_wait();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(work + 1, 1u) == gridDim.x - 1) {        // every CTA has claimed its last unit
      atomicExch(work, 0u);
      atomicExch(work + 1, 0u);
    }
  }
  // the attention kernel is released only now: released at the start, it
  // measured slower with many units per CTA (2048 units: 9 us per call)
  pdl_launch_dependents();
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

bool select_only_supported(const s3r_paged_kv& kv, int32_t budget_pages) {
  const int G = kv.num_q_heads / kv.num_kv_heads;
  return kv.dtype == S3R_BF16 && G <= 8 && budget_pages >= 1 && budget_pages <= kDfMaxBudget &&
         kv.max_pages_per_seq <= kDfMaxPages && (kv.page_size == 16 || kv.page_size == 64) &&
         (kv.head_dim == 64 || kv.head_dim == 128);
}

template <int D>
static cudaError_t launch_select_only_d(const s3r_paged_kv& kv, const AttnParams& p, int32_t* phys_out,
                                       uint32_t* work, cudaStream_t st) {
  const size_t smem = SelOnlyLay<D>::kDynBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(select_only_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // resident CTAs (once per process and head size; the kernel's resources do
  // not change)
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, select_only_kernel<D>, kDfThreads, smem);
    if (e != cudaSuccess) return e;
    per_sm = n < 1 ? 1 : n;
  }
  const int units = kv.num_seqs * kv.num_kv_heads;
  int grid = device_sm_count() * per_sm;
  if (grid > units) grid = units;
  AttnParams q = p;
  q.parts = 1;
  return launch_kernel(select_only_kernel<D>, dim3(grid), dim3(kDfThreads), smem, st, 1, q, phys_out, work);
}

cudaError_t launch_select_only(const s3r_paged_kv& kv, const AttnParams& p, int32_t* phys_out, uint32_t* work,
                               cudaStream_t st) {
  return kv.head_dim == 64 ? launch_select_only_d<64>(kv, p, phys_out, work, st)
                           : launch_select_only_d<128>(kv, p, phys_out, work, st);
}

cudaError_t launch_draft_fused(const s3r_paged_kv& kv, const DraftLaunch& dl, const AttnParams& p, cudaStream_t st) {
  if (kv.head_dim == 64)
    return launch_kernel(draft_fused_kernel<64>, dim3(dl.grid), dim3(kDfThreads), dl.smem, st, dl.parts, dl.mk,
                         dl.mv, p);
  return launch_kernel(draft_fused_kernel<128>, dim3(dl.grid), dim3(kDfThreads), dl.smem, st, dl.parts, dl.mk,
                       dl.mv, p);
}

}  // namespace s3r
