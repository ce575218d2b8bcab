// Paged attention for the S3R draft and verify steps: the fp32 kernel, the
// workspace plan shared by every attention path, and the dispatcher.
//
// S3R ("S3R: Fast and Faithful RL Rollouts via Self-Sparse Speculative
// Decoding", weekinpapers.com, Abstract) drafts with sparse attention and
// verifies with full attention over the complete KV history; both read the
// same paged cache (PagedAttention, mlsanity.com reference list).
//
// attn_f32_kernel (fp32 caches; fp32 has no exact tensor-core kind): split-KV
// on CUDA cores. A CTA owns one (sequence, KV head, split) and walks a page
// list (the selected pages for the draft, every page for verify) in 16-token
// sub-tiles with 16-byte loads; its partial softmax state is merged across
// splits by a log-sum-exp combine in the last CTA of the (sequence, KV head)
// to finish (atomic ticket, no waiting). Rows are masked causally, or by the
// round's tree (a row sees the slots of its node's ancestors and itself).
//
// launch_attention dispatches bf16 work to the tcgen05 kernels: up to 64
// packed rows (G query heads x R rows) to the token-major kernel
// (s3r_attn_tok.cu), 65-128 rows to the rows-major kernel (s3r_attn_tc.cu).
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "s3r_attn_common.cuh"
#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {


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

// ================================================================== fp32 kernel
constexpr int kF32Threads = 128;
constexpr int kF32Tok = 16;

template <int D>
__global__ void __launch_bounds__(kF32Threads) attn_f32_kernel(const AttnParams p) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) float f32_smem[];
  __shared__ int s_ticket;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const SplitGeom g = split_geom(p, b, split);
  if (g.bad_len) {
    if (split == 0) {
      if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
      write_empty_unit<float>(p, b, h, tid, kF32Threads);
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
  __shared__ unsigned long long s_tmask[64];     // tree: ancestors-or-self of each round node
  if (p.tree_parent && tid < p.R) {
    const int32_t* par = p.tree_parent + (size_t)b * p.R;
    unsigned long long m = 1ull << tid;
    int v = tid;
    for (int guard = 0; guard < 64 && v > 0; ++guard) {
      const int pv = par[v];
      if (pv < 0 || pv >= v) { flag_status(p.status, S3R_DEV_BAD_TREE); break; }
      m |= 1ull << pv;
      v = pv;
    }
    if (tid == 0 && par[0] != -1) flag_status(p.status, S3R_DEV_BAD_TREE);
    s_tmask[tid] = m;
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
        const int slot = pos - (g.L - p.R);             // >= 0: a position of the round
        const bool seen = t < ntok && (p.tree_parent ? (slot < 0 || (slot < p.R && ((s_tmask[i / p.G] >> slot) & 1ull)))
                                                      : pos <= sPos[i]);
        if (seen) {
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
      combine_partials<float>(p, b, h, unit * p.nsplit, g.nsplit_u, kF32Threads);
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

}  // namespace

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

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 148;
  return n;
}

namespace {

template <int D>
cudaError_t launch_f32(const AttnParams& p, cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)2 * p.rows * D + 2 * kF32Tok * D + (size_t)p.rows * kF32Tok + 4 * p.rows);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, p.Hkv, p.S);
  return launch_kernel(attn_f32_kernel<D>, grid, dim3(kF32Threads), smem, st, 1, p);
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
  // partial-result slots: fp32 path (unit, split); tensor-core path one slot
  // per (unit, CTA sharing it), at most units + grid
  const size_t slots_f32 = (size_t)units * pl.nsplit;
  const size_t slots_tc = (size_t)units + kMaxPersistentCtas;
  const size_t slots = kv.dtype == S3R_F32 ? slots_f32 : slots_tc;
  size_t off = kWsHeader;
  pl.off_tickets = off;
  off = align_up(off + sizeof(uint32_t) * units, 256);
  pl.off_ml = off;
  off = align_up(off + sizeof(float) * 2 * slots * prow, 256);
  pl.off_o = off;
  off = align_up(off + sizeof(float) * slots * prow * kv.head_dim, 256);
  pl.off_phys = 0;
  if (budget_pages > 0) {
    pl.off_phys = off;
    off = align_up(off + sizeof(int32_t) * units * (size_t)budget_pages, 256);
  }
  pl.ws_bytes = off;
  return pl;
}

cudaError_t launch_attention(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  *api = S3R_OK;
  if (kv.dtype == S3R_F32) {
    return kv.head_dim == 64 ? launch_f32<64>(p, st) : launch_f32<128>(p, st);
  }
  // up to 64 packed rows: token-major tiles; more: rows-major M = 128 tiles
  return p.rows <= 64 ? launch_attention_tok(kv, p, st, api) : launch_attention_tc(kv, p, st, api);
}

}  // namespace s3r
