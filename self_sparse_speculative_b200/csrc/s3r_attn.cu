// Split-KV paged attention for the S3R draft and verify steps.
//
// S3R ("S3R: Fast and Faithful RL Rollouts via Self-Sparse Speculative
// Decoding", weekinpapers.com, Abstract) drafts with sparse attention and
// verifies with full attention over the complete KV history; both read the
// same paged cache (PagedAttention, mlsanity.com reference list). One kernel
// serves both: a CTA owns one (sequence, KV head, split) and walks a page
// list - the selected pages (draft) or every page (verify) - and its partial
// softmax state is merged across splits by a log-sum-exp combine done by the
// last CTA of the (sequence, KV head) to finish (atomic ticket, no waiting).
//
// bf16 path (tcgen05): all G query heads x R rows of a (sequence, KV head)
// are packed into the rows of one MMA tile (M = 64, or 128 for more than 64
// rows), so each K/V page tile fetched from HBM feeds one dense contraction:
//   S = Q K^T  (M x 64 tokens, K = D), accumulator in tensor memory;
//   softmax on S by four warps (one TMEM lane = one packed row per thread);
//   O += P V   (M x D, K = 64 tokens), accumulator in tensor memory.
// Warp roles: warps 0-3 softmax/epilogue, warp 4 TMA producer, warp 5 MMA
// issuer + TMEM owner. K/V tiles arrive by TMA (3-D tensor map over the
// cache, 128-byte swizzle, one box per page and 64-channel half) into a
// 2-stage ring; S is double-buffered in TMEM so QK(j+1) overlaps softmax(j).
// The running max is rescaled lazily (only when it grows by more than 2^8),
// which leaves the result exact: O and l always share one reference.
//
// fp32 path: the same split/combine structure on CUDA cores with 16-byte
// vector loads (fp32 has no exact tensor-core kind).
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kTcThreads = 192;     // 4 softmax warps + producer + MMA
constexpr int kStages = 2;
constexpr float kRescaleTau = 8.0f; // log2 units
constexpr float kLn2 = 0.6931471805599453f;

// ------------------------------------------------------------------ combine
template <typename OutT>
__device__ __forceinline__ void store_out4(OutT* dst, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store_out4<__nv_bfloat16>(__nv_bfloat16* dst, float a, float b, float c, float d) {
  uint2 v = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
  *reinterpret_cast<uint2*>(dst) = v;
}
template <>
__device__ __forceinline__ void store_out4<float>(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}

__device__ __forceinline__ size_t out_row_offset(const AttnParams& p, int b, int h, int i) {
  const int r = i / p.G, g = i - (i / p.G) * p.G;
  return ((size_t)(b * p.R + r) * p.Hq + (size_t)h * p.G + g);
}

// Merge the nsplit_u partial states of unit (b, h) into the final output.
// Runs on `nthreads` consecutive threads starting at thread 0.
template <typename OutT>
__device__ void combine_unit(const AttnParams& p, int b, int h, int nsplit_u, int nthreads) {
  const int unit = b * p.Hkv + h;
  const int D4 = p.D / 4;
  for (int idx = threadIdx.x; idx < p.rows * D4; idx += nthreads) {
    const int i = idx / D4, d4 = idx - (idx / D4) * D4;
    float M = -INFINITY;
    for (int s = 0; s < nsplit_u; ++s) {
      const float m = __ldcg(p.part_ml + (((size_t)unit * p.nsplit + s) * p.rows + i) * 2);
      M = fmaxf(M, m);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float Ls = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < nsplit_u; ++s) {
        const size_t pi = ((size_t)unit * p.nsplit + s) * p.rows + i;
        const float m = __ldcg(p.part_ml + pi * 2), l = __ldcg(p.part_ml + pi * 2 + 1);
        if (m == -INFINITY || l == 0.f) continue;
        const float w = exp2f(m - M);
        Ls += l * w;
        const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + pi * p.D) + d4);
        acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    const size_t orow = out_row_offset(p, b, h, i);
    store_out4<OutT>(static_cast<OutT*>(p.out) + orow * p.D + d4 * 4, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (d4 == 0 && p.lse) p.lse[orow] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
  }
}

// Outputs of a unit whose context length is invalid: zeros and lse = -inf.
template <typename OutT>
__device__ void write_empty_unit(const AttnParams& p, int b, int h, int nthreads) {
  const int D4 = p.D / 4;
  for (int idx = threadIdx.x; idx < p.rows * D4; idx += nthreads) {
    const int i = idx / D4, d4 = idx - (idx / D4) * D4;
    const size_t orow = out_row_offset(p, b, h, i);
    store_out4<OutT>(static_cast<OutT*>(p.out) + orow * p.D + d4 * 4, 0.f, 0.f, 0.f, 0.f);
    if (d4 == 0 && p.lse) p.lse[orow] = -INFINITY;
  }
}

// Geometry of one CTA's share of a unit.
struct SplitGeom {
  int L, n_b, total_pages, nsplit_u, pg0, npg;
  bool bad_len;
};
__device__ __forceinline__ SplitGeom split_geom(const AttnParams& p, int b, int split) {
  SplitGeom g;
  g.L = p.context_lens[b];
  g.bad_len = (g.L < p.R) || (g.L > p.max_pages * p.P) || (g.L < 1);
  g.n_b = g.bad_len ? 0 : (g.L + p.P - 1) / p.P;
  g.total_pages = p.page_list ? min(p.budget, g.n_b) : g.n_b;
  g.nsplit_u = (g.total_pages + p.chunk_pages - 1) / p.chunk_pages;
  g.pg0 = split * p.chunk_pages;
  g.npg = min(p.chunk_pages, g.total_pages - g.pg0);
  return g;
}

// Logical and physical page of list entry k (k < npg) of this CTA; -1 when
// missing or out of range (recorded in the status word).
__device__ __forceinline__ void resolve_page(const AttnParams& p, int b, int h, const SplitGeom& g, int k,
                                             int32_t* lp_out, int32_t* phys_out) {
  int lp = p.page_list ? p.page_list[((size_t)b * p.Hkv + h) * p.budget + g.pg0 + k] : g.pg0 + k;
  int phys = -1;
  if (lp >= 0 && lp < g.n_b) {
    phys = p.block_table[(size_t)b * p.max_pages + lp];
    if (phys < 0 || phys >= p.num_pages_total) {
      flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      phys = -1;
    }
  } else {
    flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
    lp = -1;
  }
  *lp_out = lp;
  *phys_out = phys;
}

// ================================================================== tcgen05 kernel
template <int M, int D>
struct TcLayout {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQBytes = M * D * 2;
  static constexpr uint32_t kPBytes = M * 128;                // 64 tokens x bf16
  static constexpr uint32_t kTileBytes = kStageTokens * D * 2; // K or V of one stage
  static constexpr uint32_t kOffP = kQBytes;
  static constexpr uint32_t kOffKV = kOffP + 2 * kPBytes;
  static constexpr uint32_t kDynBytes = kOffKV + kStages * 2 * kTileBytes;
  static constexpr uint32_t kTmemCols = 256;                   // S0 | S1 | O
};

template <int M, int D>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const AttnParams p) {
  using Lay = TcLayout<M, D>;
  extern __shared__ __align__(1024) uint8_t dyn_raw[];
  uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t s_bar[2 * kStages + 7];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_ticket;
  __shared__ int32_t s_lp[kMaxSplitPages];
  __shared__ int32_t s_phys[kMaxSplitPages];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const SplitGeom g = split_geom(p, b, split);
  if (g.bad_len) {
    if (split == 0) {
      if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
      write_empty_unit<__nv_bfloat16>(p, b, h, kTcThreads);
    }
    return;
  }
  if (split >= g.nsplit_u) return;
  const int ppt = kStageTokens / p.P;                 // pages per stage
  const int nstages = (g.npg + ppt - 1) / ppt;

  const uint32_t bar_full = smem_addr(&s_bar[0]);
  const uint32_t bar_empty = smem_addr(&s_bar[kStages]);
  const uint32_t bar_sfull = smem_addr(&s_bar[2 * kStages]);      // 2
  const uint32_t bar_pfull = smem_addr(&s_bar[2 * kStages + 2]);  // 2
  const uint32_t bar_odone = smem_addr(&s_bar[2 * kStages + 4]);
  const uint32_t bar_td = smem_addr(&s_bar[2 * kStages + 5]);
  auto bar = [](uint32_t base, int i) { return base + 8u * i; };

  uint8_t* sQ = dyn;
  uint8_t* sP = dyn + Lay::kOffP;
  uint8_t* sKV = dyn + Lay::kOffKV;
  const uint32_t aQ = smem_addr(sQ), aP = smem_addr(sP), aKV = smem_addr(sKV);

  // ---- setup
  if (warp == 5) {
    tmem_alloc(smem_addr(&s_tmem), Lay::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(bar(bar_full, i), 1); mbar_init(bar(bar_empty, i), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(bar(bar_sfull, i), 1); mbar_init(bar(bar_pfull, i), 128); }
    mbar_init(bar_odone, 1);
    mbar_init(bar_td, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) { prefetch_tensormap(&tmK); prefetch_tensormap(&tmV); }
  for (int k = tid; k < g.npg; k += kTcThreads) resolve_page(p, b, h, g, k, &s_lp[k], &s_phys[k]);
  if (tid < 128) {
    // Q rows -> tile rows, bf16, K-major 128-byte swizzle; padding rows zero
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
    constexpr int kChunks = D / 8;                   // 16-byte chunks per row
    for (int idx = tid; idx < M * kChunks; idx += 128) {
      const int slot = idx / kChunks, c16 = idx - (idx / kChunks) * kChunks;
      const int i = (M == 64) ? 4 * (slot & 15) + (slot >> 4) : 4 * (slot & 31) + (slot >> 5);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (i < p.rows) v = *reinterpret_cast<const uint4*>(q + out_row_offset(p, b, h, i) * D + c16 * 8);
      const int half = c16 >> 3, c = c16 & 7;
      *reinterpret_cast<uint4*>(sQ + half * (M * 128) + slot * 128 + ((c ^ (slot & 7)) << 4)) = v;
    }
    for (int idx = tid; idx < (int)(2 * Lay::kPBytes / 16); idx += 128)
      reinterpret_cast<uint4*>(sP)[idx] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 4) {
    // ================= TMA producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int issued = 0;
      for (int j = 0; j < nstages; ++j) {
        const int st = j % kStages;
        if (!mbar_wait(bar(bar_empty, st), ((j / kStages) & 1) ^ 1, &s_abort, p.status)) break;
        int nreal = 0;
        for (int pp = 0; pp < ppt; ++pp) {
          const int k = j * ppt + pp;
          if (k < g.npg && s_phys[k] >= 0) ++nreal;
        }
        mbar_arrive_expect_tx(bar(bar_full, st), (uint32_t)nreal * Lay::kHalves * 2u * (uint32_t)p.P * 128u);
        const uint32_t dK = aKV + st * 2 * Lay::kTileBytes, dV = dK + Lay::kTileBytes;
        for (int pp = 0; pp < ppt; ++pp) {
          const int k = j * ppt + pp;
          if (k >= g.npg || s_phys[k] < 0) continue;
          const int z = s_phys[k] * p.Hkv + h;
          for (int hh = 0; hh < Lay::kHalves; ++hh) {
            const uint32_t off = hh * (kStageTokens * 128) + pp * (p.P * 128);
            tma_load_3d(dK + off, &tmK, bar(bar_full, st), hh * 64, 0, z, pol);
            tma_load_3d(dV + off, &tmV, bar(bar_full, st), hh * 64, 0, z, pol);
          }
        }
        issued = j + 1;
      }
      for (int j = max(0, issued - kStages); j < issued; ++j)
        mbar_wait_drain(bar(bar_full, j % kStages), (j / kStages) & 1, p.status);
    }
  } else if (warp == 5) {
    // ================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(M, kStageTokens, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(M, D, false, true);
      for (int j = 0; j <= nstages; ++j) {
        if (j < nstages) {
          const int st = j % kStages;
          if (!mbar_wait(bar(bar_full, st), (j / kStages) & 1, &s_abort, p.status)) break;
          tc_fence_after();
          const uint32_t kb = aKV + st * 2 * Lay::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int hh = kk >> 2, sub = kk & 3;
            const uint64_t a = smem_desc_sw128(aQ + hh * (M * 128) + sub * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kb + hh * (kStageTokens * 128) + sub * 32, 16, 1024);
            umma_f16(tS + (j & 1) * kStageTokens, a, bd, idQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(bar_sfull, j & 1));
        }
        if (j >= 1) {
          const int jp = j - 1, stp = jp % kStages;
          if (!mbar_wait(bar(bar_pfull, jp & 1), (jp >> 1) & 1, &s_abort, p.status)) break;
          tc_fence_after();
          const uint32_t vb = aKV + stp * 2 * Lay::kTileBytes + Lay::kTileBytes;
          const uint32_t pb = aP + (jp & 1) * Lay::kPBytes;
#pragma unroll
          for (int kk = 0; kk < kStageTokens / 16; ++kk) {
            const uint64_t a = smem_desc_sw128(pb + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(vb + kk * (16 * 128), kStageTokens * 128, 1024);
            umma_f16(tO, a, bd, idPV, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar(bar_empty, stp));
          umma_commit(bar_odone);
        }
      }
      umma_commit(bar_td);
    }
  } else {
    // ================= softmax warps (tid 0..127)
    const int q4 = warp;
    const int slot = (M == 64) ? (lane < 16 ? 16 * q4 + lane : -1) : 32 * q4 + lane;
    const int i = 4 * lane + q4;                       // packed row of this thread's slot
    const bool valid_row = slot >= 0 && i < p.rows;
    const int r = valid_row ? i / p.G : 0;
    const int qpos = g.L - p.R + r;                    // this row's position
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nstages; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(bar_sfull, sb), (j >> 1) & 1, &s_abort, p.status))) { ok = false; break; }
      tc_fence_after();
      float s[kStageTokens];
      tmem_ld32(tS + lane_base + sb * kStageTokens, s);
      tmem_ld32(tS + lane_base + sb * kStageTokens + 32, s + 32);
      tmem_wait_ld();

      // token validity of this stage: positions lp*P + t must be < L, and
      // <= the row position (causal); pages may be missing at the end
      const int k0 = j * ppt;
      bool any_invalid = false;      // some token of the stage must be zeroed in V
      bool need_mask = false;        // some column is masked for some row
      for (int pp = 0; pp < ppt; ++pp) {
        const int k = k0 + pp;
        if (k >= g.npg || s_phys[k] < 0) { any_invalid = true; continue; }
        const int last_pos = s_lp[k] * p.P + p.P - 1;
        if (last_pos >= g.L) any_invalid = true;
        if (last_pos > g.L - p.R) need_mask = true;
      }
      need_mask |= any_invalid;
      float mx = -INFINITY;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < kStageTokens; ++c) {
          const int k = k0 + c / p.P;
          bool v = false;
          if (k < g.npg && s_phys[k] >= 0) {
            const int pos = s_lp[k] * p.P + (c % p.P);
            v = pos < g.L && pos <= qpos;
          }
          s[c] = v ? s[c] * p.scale_log2 : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kStageTokens; ++c) { s[c] *= p.scale_log2; mx = fmaxf(mx, s[c]); }
      }
      // lazy running-max update
      float alpha = 1.f;
      bool rescale = false;
      if (valid_row) {
        if (m_run == -INFINITY) {
          m_run = mx;                                   // O rows are still zero
        } else if (mx > m_run + kRescaleTau) {
          alpha = ex2(m_run - mx);
          m_run = mx;
          l_run *= alpha;
          rescale = true;
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // P = 2^(s - m), rounded to bf16; l sums the rounded values
      uint32_t pk[kStageTokens / 2];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < kStageTokens; c += 2) {
        const float e0 = ex2(s[c] - m_use), e1 = ex2(s[c + 1] - m_use);
        pk[c / 2] = pack_bf16x2(e0, e1);
        const __nv_bfloat162 rb = *reinterpret_cast<__nv_bfloat162*>(&pk[c / 2]);
        lsum += __low2float(rb) + __high2float(rb);
      }
      if (valid_row) l_run += lsum;

      // PV(j-1) must be complete before O is rescaled or P[sb] is rewritten
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(bar_odone, (j - 1) & 1, &s_abort, p.status))) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tmem_ld32(tO + lane_base + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= alpha;
          tmem_st32(tO + lane_base + c0, o);
        }
        tmem_wait_st();
      }
      if (any_invalid) {
        // zero the V rows of tokens that do not exist (beyond L, missing
        // pages) so that 0 * garbage cannot reach O
        if (!__all_sync(0xffffffffu, mbar_wait(bar(bar_full, j % kStages), (j / kStages) & 1, &s_abort, p.status))) { ok = false; break; }
        uint8_t* sV = sKV + (j % kStages) * 2 * Lay::kTileBytes + Lay::kTileBytes;
        for (int idx = tid; idx < kStageTokens * Lay::kHalves * 8; idx += 128) {
          const int t = idx / (Lay::kHalves * 8);
          const int rem = idx - t * (Lay::kHalves * 8);
          const int hh = rem >> 3, c = rem & 7;
          const int k = k0 + t / p.P;
          bool v = false;
          if (k < g.npg && s_phys[k] >= 0) v = s_lp[k] * p.P + (t % p.P) < g.L;
          if (!v) *reinterpret_cast<uint4*>(sV + hh * (kStageTokens * 128) + t * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (valid_row) {
        uint8_t* prow = sP + sb * Lay::kPBytes + slot * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ (slot & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(bar_pfull, sb));
    }
    // ---- epilogue
    if (ok && nstages > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_odone, (nstages - 1) & 1, &s_abort, p.status));
    tc_fence_after();
    const bool single = (g.nsplit_u == 1);
    const int unit = b * p.Hkv + h;
    const size_t pi = ((size_t)unit * p.nsplit + split) * p.rows + (valid_row ? i : 0);
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    for (int c0 = 0; c0 < D; c0 += 32) {
      float o[32];
      tmem_ld32(tO + lane_base + c0, o);
      tmem_wait_ld();
      if (!valid_row) continue;
      if (!ok || nstages == 0) {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0.f;
      }
      if (single) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + out_row_offset(p, b, h, i) * D + c0;
#pragma unroll
        for (int c = 0; c < 32; c += 8)
          *reinterpret_cast<uint4*>(dst + c) =
              make_uint4(pack_bf16x2(o[c] * inv_l, o[c + 1] * inv_l), pack_bf16x2(o[c + 2] * inv_l, o[c + 3] * inv_l),
                         pack_bf16x2(o[c + 4] * inv_l, o[c + 5] * inv_l), pack_bf16x2(o[c + 6] * inv_l, o[c + 7] * inv_l));
      } else {
        float* dst = p.part_o + pi * D + c0;
#pragma unroll
        for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      }
    }
    if (valid_row) {
      if (!ok) { m_run = -INFINITY; l_run = 0.f; }
      if (single) {
        if (p.lse) p.lse[out_row_offset(p, b, h, i)] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      } else {
        p.part_ml[pi * 2] = l_run > 0.f ? m_run : -INFINITY;
        p.part_ml[pi * 2 + 1] = l_run;
      }
    }
    if (!single) {
      __threadfence();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) s_ticket = atomicAdd(p.tickets + unit, 1u);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (s_ticket == g.nsplit_u - 1) {
        __threadfence();
        combine_unit<__nv_bfloat16>(p, b, h, g.nsplit_u, 128);
        if (tid == 0) p.tickets[unit] = 0u;
      }
    }
  }

  // ---- teardown: every role is done; wait for the MMAs, free TMEM
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    if (lane == 0) mbar_wait_drain(bar_td, 0, p.status);
    __syncwarp();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

// ================================================================== fp32 kernel
constexpr int kF32Threads = 128;
constexpr int kF32Tok = 16;

template <int D>
__global__ void __launch_bounds__(kF32Threads) attn_f32_kernel(const AttnParams p) {
  extern __shared__ __align__(16) float f32_smem[];
  __shared__ int s_ticket;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const SplitGeom g = split_geom(p, b, split);
  if (g.bad_len) {
    if (split == 0) {
      if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
      write_empty_unit<float>(p, b, h, kF32Threads);
    }
    return;
  }
  if (split >= g.nsplit_u) return;
  const int rows = p.rows;
  float* sQ = f32_smem;                       // [rows, D]
  float* sO = sQ + rows * D;                  // [rows, D]
  float* sK = sO + rows * D;                  // [16, D]
  float* sV = sK + kF32Tok * D;               // [16, D]
  float* sS = sV + kF32Tok * D;               // [rows, 16]
  float* sM = sS + rows * kF32Tok;            // [rows]
  float* sL = sM + rows;                      // [rows]
  float* sA = sL + rows;                      // [rows]
  int* sPos = reinterpret_cast<int*>(sA + rows);  // [rows]

  const float* q = static_cast<const float*>(p.q);
  for (int idx = tid; idx < rows * D; idx += kF32Threads) {
    const int i = idx / D, d = idx - (idx / D) * D;
    sQ[idx] = q[out_row_offset(p, b, h, i) * D + d];
    sO[idx] = 0.f;
  }
  for (int i = tid; i < rows; i += kF32Threads) {
    sM[i] = -INFINITY;
    sL[i] = 0.f;
    sPos[i] = g.L - p.R + i / p.G;
  }
  __syncthreads();
  const float* kc = static_cast<const float*>(p.k_cache);
  const float* vc = static_cast<const float*>(p.v_cache);
  for (int k = 0; k < g.npg; ++k) {
    int lp, phys;
    resolve_page(p, b, h, g, k, &lp, &phys);
    if (phys < 0) continue;
    const int valid = min(p.P, g.L - lp * p.P);
    for (int t0 = 0; t0 < valid; t0 += kF32Tok) {
      const int ntok = min(kF32Tok, valid - t0);
      const size_t base = (((size_t)phys * p.Hkv + h) * p.P + t0) * D;
      for (int idx = tid; idx < kF32Tok * D / 4; idx += kF32Threads) {
        const int t = idx / (D / 4);
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
        if (t < ntok) {
          kv = __ldg(reinterpret_cast<const float4*>(kc + base) + idx);
          vv = __ldg(reinterpret_cast<const float4*>(vc + base) + idx);
        }
        reinterpret_cast<float4*>(sK)[idx] = kv;
        reinterpret_cast<float4*>(sV)[idx] = vv;
      }
      __syncthreads();
      for (int idx = tid; idx < rows * kF32Tok; idx += kF32Threads) {
        const int i = idx / kF32Tok, t = idx - (idx / kF32Tok) * kF32Tok;
        const int pos = lp * p.P + t0 + t;
        float sc = -INFINITY;
        if (t < ntok && pos <= sPos[i]) {
          const float4* a = reinterpret_cast<const float4*>(sQ + i * D);
          const float4* kk = reinterpret_cast<const float4*>(sK + t * D);
          float acc = 0.f;
#pragma unroll 8
          for (int d = 0; d < D / 4; ++d) {
            const float4 x = a[d], y = kk[d];
            acc = fmaf(x.x, y.x, acc); acc = fmaf(x.y, y.y, acc);
            acc = fmaf(x.z, y.z, acc); acc = fmaf(x.w, y.w, acc);
          }
          sc = acc * p.scale_log2;
        }
        sS[idx] = sc;
      }
      __syncthreads();
      for (int i = tid; i < rows; i += kF32Threads) {
        float mx = -INFINITY;
        for (int t = 0; t < kF32Tok; ++t) mx = fmaxf(mx, sS[i * kF32Tok + t]);
        const float m_old = sM[i];
        const float m_new = fmaxf(m_old, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - m_use);
        float sum = 0.f;
        for (int t = 0; t < kF32Tok; ++t) {
          const float e = exp2f(sS[i * kF32Tok + t] - m_use);
          sS[i * kF32Tok + t] = e;
          sum += e;
        }
        sL[i] = sL[i] * alpha + sum;
        sM[i] = m_new;
        sA[i] = alpha;
      }
      __syncthreads();
      for (int idx = tid; idx < rows * D; idx += kF32Threads) {
        const int i = idx / D, d = idx - (idx / D) * D;
        float acc = sO[idx] * sA[i];
        for (int t = 0; t < kF32Tok; ++t) acc = fmaf(sS[i * kF32Tok + t], sV[t * D + d], acc);
        sO[idx] = acc;
      }
      __syncthreads();
    }
  }
  const bool single = (g.nsplit_u == 1);
  const int unit = b * p.Hkv + h;
  for (int idx = tid; idx < rows * D; idx += kF32Threads) {
    const int i = idx / D, d = idx - (idx / D) * D;
    if (single) {
      const float l = sL[i];
      static_cast<float*>(p.out)[out_row_offset(p, b, h, i) * D + d] = l > 0.f ? sO[idx] / l : 0.f;
    } else {
      p.part_o[(((size_t)unit * p.nsplit + split) * rows + i) * D + d] = sO[idx];
    }
  }
  for (int i = tid; i < rows; i += kF32Threads) {
    const float l = sL[i], m = sM[i];
    if (single) {
      if (p.lse) p.lse[out_row_offset(p, b, h, i)] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    } else {
      const size_t pi = ((size_t)unit * p.nsplit + split) * rows + i;
      p.part_ml[pi * 2] = l > 0.f ? m : -INFINITY;
      p.part_ml[pi * 2 + 1] = l;
    }
  }
  if (!single) {
    __threadfence();
    __syncthreads();
    if (tid == 0) s_ticket = atomicAdd(p.tickets + unit, 1u);
    __syncthreads();
    if (s_ticket == g.nsplit_u - 1) {
      __threadfence();
      combine_unit<float>(p, b, h, g.nsplit_u, kF32Threads);
      if (tid == 0) p.tickets[unit] = 0u;
    }
  }
}

// ================================================================== host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D map over a [pages * Hkv, P, D] bf16 cache, box = 64 channels x P tokens x 1.
bool make_cache_map(CUtensorMap* map, const void* base, const s3r_paged_kv& kv) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kv.head_dim, (cuuint64_t)kv.page_size,
                              (cuuint64_t)kv.num_pages_total * (cuuint64_t)kv.num_kv_heads};
  const cuuint64_t strides[2] = {(cuuint64_t)kv.head_dim * 2, (cuuint64_t)kv.head_dim * kv.page_size * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)kv.page_size, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int M, int D>
cudaError_t launch_tc(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  CUtensorMap mk, mv;
  if (!make_cache_map(&mk, kv.k_cache, kv) || !make_cache_map(&mv, kv.v_cache, kv)) {
    *api = S3R_ERR_CUDA;
    return cudaErrorInvalidValue;
  }
  const size_t smem = TcLayout<M, D>::kDynBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<M, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, p.Hkv, p.S);
  attn_tc_kernel<M, D><<<grid, kTcThreads, smem, st>>>(mk, mv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_f32(const AttnParams& p, cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)2 * p.rows * D + 2 * kF32Tok * D + (size_t)p.rows * kF32Tok + 4 * p.rows);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, p.Hkv, p.S);
  attn_f32_kernel<D><<<grid, kF32Threads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

AttnPlan plan_attention(const s3r_paged_kv& kv, int32_t rows, int32_t budget_pages) {
  AttnPlan pl{};
  const int G = kv.num_q_heads / kv.num_kv_heads;
  const int prow = G * rows;
  const int units = kv.num_seqs * kv.num_kv_heads;
  const int max_list = budget_pages > 0 ? (budget_pages < kv.max_pages_per_seq ? budget_pages : kv.max_pages_per_seq)
                                        : kv.max_pages_per_seq;
  // pages per split: a multiple of the pages per 64-token stage, sized so that
  // the grid holds about 8 CTAs per SM, each CTA with at least 4 stages
  const int ppt = kv.page_size < kStageTokens ? kStageTokens / kv.page_size : 1;
  const int stages = (max_list + ppt - 1) / ppt;
  const int target_ctas = 148 * 8;
  int nsplit = (target_ctas + units - 1) / units;
  const int max_split_by_len = (stages + 3) / 4;
  if (nsplit > max_split_by_len) nsplit = max_split_by_len;
  if (nsplit < 1) nsplit = 1;
  int chunk_stages = (stages + nsplit - 1) / nsplit;
  const int cap = kMaxSplitPages / ppt;
  if (chunk_stages > cap) chunk_stages = cap;
  if (chunk_stages < 1) chunk_stages = 1;
  pl.chunk_pages = chunk_stages * ppt;
  pl.nsplit = (max_list + pl.chunk_pages - 1) / pl.chunk_pages;
  if (pl.nsplit < 1) pl.nsplit = 1;
  size_t off = kWsHeader;
  pl.off_tickets = off;
  off = align_up(off + sizeof(uint32_t) * units, 256);
  pl.off_ml = off;
  off = align_up(off + sizeof(float) * 2 * (size_t)units * pl.nsplit * prow, 256);
  pl.off_o = off;
  off = align_up(off + sizeof(float) * (size_t)units * pl.nsplit * prow * kv.head_dim, 256);
  pl.ws_bytes = off;
  return pl;
}

cudaError_t launch_attention(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  *api = S3R_OK;
  if (kv.dtype == S3R_F32) {
    return kv.head_dim == 64 ? launch_f32<64>(p, st) : launch_f32<128>(p, st);
  }
  const bool small = p.rows <= 64;
  if (kv.head_dim == 64) return small ? launch_tc<64, 64>(kv, p, st, api) : launch_tc<128, 64>(kv, p, st, api);
  return small ? launch_tc<64, 128>(kv, p, st, api) : launch_tc<128, 128>(kv, p, st, api);
}

}  // namespace s3r
