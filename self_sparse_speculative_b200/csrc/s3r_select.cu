// Query-aware page selection for the sparse draft (Quest-style scoring on
// the mlsanity.com page's reference list; S3R page, Abstract, "uses sparse
// attention to propose tokens").
//
// One thread-block cluster of CL CTAs per (sequence, KV head):
//   1. every CTA scores its share of the pages p < n_b with the float64 bound
//        s(p) = sum_g sum_d max(q[g,d] * kmin[p,d], q[g,d] * kmax[p,d])
//      over the G query heads of the group. Per channel the sum over g folds
//      into two weights (exact in real arithmetic, for any kmin, kmax):
//        sum_g max(q_g a, q_g b) = A max(a, b) + B min(a, b),
//        A = sum_g max(q_g, 0),  B = sum_g min(q_g, 0),
//      so a page costs 2 D float64 multiply-adds whatever G is (one warp per
//      page, eight pages in flight per warp). The tail page n_b - 1, whose
//      summary still changes while the sequence decodes, is summarised from K
//      (staged by cp.async before the dependency wait) and scored last. The
//      pages' order-preserving 64-bit keys and physical ids go into the shared
//      memory of the cluster's first CTA (distributed shared memory);
//   2. that CTA radix-selects the budget-th largest key (8-bit digits from the
//      first byte in which the keys differ: shared-memory histogram, one-warp
//      scan of the 256 bins), stopping as soon as the boundary bin holds
//      exactly the keys still needed (a rank count of every key against all
//      others measured slower);
//   3. it keeps the keys above the boundary plus the lowest-index pages on it,
//      writes them in ascending page order with block-wide prefix sums (the
//      logical ids to `selected`, the physical ids for the attention kernel),
//      and prefetches the first selected pages' K and V into L2.
#include <cuda_bf16.h>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

__device__ __forceinline__ unsigned long long order_key(double x) {
  unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}


// Exclusive prefix sum over the CTA (kSelThreads threads); also returns the total.
__device__ int block_exclusive_scan(int v, int* total, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kSelWarps ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelWarps) s_warp[lane] = w;     // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
  *total = s_warp[kSelWarps - 1];
  __syncthreads();
  return before;
}

struct SelParams {
  const void* q;            // [S, Hq, D]
  const void* kmin;
  const void* kmax;         // [num_pages_total, Hkv, D]
  const void* k_cache;      // [num_pages_total, Hkv, P, D] (the tail page's summary is taken from it)
  const void* v_cache;      // [num_pages_total, Hkv, P, D] (only prefetched into L2)
  const int32_t* block_table;
  const int32_t* context_lens;
  int32_t* selected;        // [S, Hkv, budget]
  int32_t* selected_phys;   // [S, Hkv, budget] physical ids of the selected pages (-1: none)
  int32_t S, Hq, Hkv, G, D, P, max_pages, num_pages_total, budget;
  int32_t elt;              // bytes per K/V element
  uint32_t* status;
};

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// 16-byte global -> shared copy through L2 (cp.async; completion per thread
// by commit groups)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_cluster_u32(uint32_t local_addr, uint32_t rank, uint32_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(remote), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_u64(uint32_t local_addr, uint32_t rank, unsigned long long v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("st.shared::cluster.u64 [%0], %1;" :: "r"(remote), "l"(v) : "memory");
}

// A lane's CPL channels of one summary row, as loaded (packed) and unpacked.
template <typename T, int CPL> struct RawRow;
template <> struct RawRow<__nv_bfloat16, 4> {
  using type = uint2;
  __device__ static void unpack(const uint2& u, float* v) {
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  }
};
template <> struct RawRow<__nv_bfloat16, 2> {
  using type = uint32_t;
  __device__ static void unpack(const uint32_t& u, float* v) {
    v[0] = __uint_as_float(u << 16); v[1] = __uint_as_float(u & 0xFFFF0000u);
  }
};
template <> struct RawRow<float, 4> {
  using type = float4;
  __device__ static void unpack(const float4& u, float* v) { v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w; }
};
template <> struct RawRow<float, 2> {
  using type = float2;
  __device__ static void unpack(const float2& u, float* v) { v[0] = u.x; v[1] = u.y; }
};

// A 16-byte vector of K as floats (8 bf16 or 4 fp32 values).
template <typename T> __device__ __forceinline__ void unpack16(const uint4& u, float* v);
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* v) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) { v[2 * k] = __uint_as_float(w[k] << 16); v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u); }
}
template <> __device__ __forceinline__ void unpack16<float>(const uint4& u, float* v) {
  v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
}

__device__ __forceinline__ float load_scalar(const __nv_bfloat16* p, int i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float load_scalar(const float* p, int i) { return p[i]; }

// Pages per warp and round: 8, or 4 when a page's two summary rows exceed
// 512 bytes (fp32, D = 128).
template <typename T, int CPL>
__host__ __device__ constexpr int sel_unroll() { return sizeof(T) * CPL * 32 * 2 > 512 ? 4 : 8; }

// Dynamic shared memory: keys [max_pages] (u64), physical page ids
// [max_pages] (int), then the tail page's K [P, D] (16-byte aligned).
__host__ __device__ inline size_t sel_off_tailk(int max_pages) { return ((size_t)max_pages * 12 + 15) / 16 * 16; }
inline size_t sel_smem_bytes(int max_pages, int P, int D, int elt) {
  return sel_off_tailk(max_pages) + (size_t)P * D * elt;
}

// The attention kernel that follows streams the selected pages in list
// order; the first kPrefetchPages of them (K and V) are prefetched into L2 as
// soon as they are known, so its first stages do not wait for DRAM.
constexpr int kPrefetchPages = 8;
__device__ __forceinline__ void prefetch_page(const SelParams& p, int phys, int h) {
  if (phys < 0 || phys >= p.num_pages_total) return;
  const uint32_t bytes = static_cast<uint32_t>(p.P * p.D) * p.elt;
  const size_t off = ((size_t)phys * p.Hkv + h) * bytes;
  bulk_prefetch_l2(static_cast<const char*>(p.k_cache) + off, bytes);
  bulk_prefetch_l2(static_cast<const char*>(p.v_cache) + off, bytes);
}

// MINB: CTAs per SM the registers are bounded for (2, or 4 for launches with
// more units than two per SM hold).
template <typename T, int CPL, int MINB>
__global__ void __launch_bounds__(kSelThreads, MINB) select_kernel(const SelParams p) {
  extern __shared__ unsigned long long s_keys[];          // [max_pages] keys, then [max_pages] page ids
  __shared__ __align__(16) double s_ab[2][128];         // A, B per channel
  __shared__ __align__(16) float s_tail[2][128];       // min / max of the tail page (this CTA's, if any)
  __shared__ float s_tpart[2][kSelWarps][128];          // per-warp partial min / max of the tail page
  __shared__ unsigned long long s_kred[2][kSelWarps];   // key min / max per warp
  __shared__ unsigned int s_hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_k, s_done, s_shift, s_start;
  __shared__ int s_warp[kSelWarps];

  pdl_launch_dependents();
  const int h = blockIdx.y, b = blockIdx.z;
  const uint32_t rank = cluster_rank();
  const int ncta = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* out = p.selected + ((size_t)b * p.Hkv + h) * p.budget;
  int32_t* out_phys = p.selected_phys + ((size_t)b * p.Hkv + h) * p.budget;
  // the group's query values first (they depend on nothing), so their loads
  // overlap the context length -> page id -> tail K chain below
  const T* qp = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)h * p.G) * p.D;
  float qv[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) qv[g] = (tid < p.D && g < p.G) ? load_scalar(qp, g * p.D + tid) : 0.f;
  // every decision before the cluster barriers is uniform over the cluster
  const int L = p.context_lens[b];
  if (L < 1 || L > p.max_pages * p.P) {
    pdl_wait();
    if (rank == 0) {
      if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
      for (int k = tid; k < p.budget; k += kSelThreads) { out[k] = -1; out_phys[k] = -1; }
    }
    return;
  }
  const int n_b = (L + p.P - 1) / p.P;
  if (n_b <= p.budget) {
    pdl_wait();
    if (rank == 0)
      for (int k = tid; k < p.budget; k += kSelThreads) {
        const int ph = k < n_b ? p.block_table[(size_t)b * p.max_pages + k] : -1;
        out[k] = k < n_b ? k : -1;
        out_phys[k] = ph;
        if (k < kPrefetchPages) prefetch_page(p, ph, h);
      }
    return;
  }
  // announce this CTA to the cluster now; wait for the others only before
  // touching the first CTA's shared memory
  cluster_arrive();

  // ---- 1. scores of pages [beg, end) into this CTA's own key array
  const int per = (n_b + ncta - 1) / ncta;
  const int beg = min(n_b, (int)rank * per), end = min(n_b, beg + per);
  const T* kmn = static_cast<const T*>(p.kmin);
  const T* kmx = static_cast<const T*>(p.kmax);
  // This CTA's page ids and the weights A, B of every channel (inputs, so
  // read before the dependency wait). The tail page n_b - 1 is the only one
  // whose summary changes while a sequence decodes: the CTA that scores it
  // takes its min / max over the valid tokens straight from K.
  const int tail = n_b - 1;
  const bool has_tail = beg <= tail && tail < end;
  const int tail_phys = has_tail ? p.block_table[(size_t)b * p.max_pages + tail] : -1;
  int* s_phys = reinterpret_cast<int*>(s_keys + p.max_pages);
  for (int pg = beg + tid; pg < end; pg += kSelThreads) s_phys[pg] = p.block_table[(size_t)b * p.max_pages + pg];
  if (tid < p.D) {
    double a = 0.0, z = 0.0;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const double v = static_cast<double>(qv[g]);
      if (v > 0.0) a += v; else z += v;                 // zero padding adds nothing
    }
    s_ab[0][tid] = a;
    s_ab[1][tid] = z;
  }
  // The tail page's valid tokens of K go to shared memory by cp.async now;
  // they are reduced to the page's min / max after the other pages are scored.
  constexpr int VEC = 16 / sizeof(T);
  const int chunks = p.D / VEC, groups = kSelThreads / chunks;
  const int tc = tid % chunks, tgrp = tid / chunks;
  constexpr int kMaxPer = 8;                            // tokens per thread: P <= groups * 8
  const bool tail_ok = has_tail && tail_phys >= 0 && tail_phys < p.num_pages_total;
  const int valid = L - tail * p.P;
  const T* s_tk = reinterpret_cast<const T*>(reinterpret_cast<const uint8_t*>(s_keys) + sel_off_tailk(p.max_pages));
  if (tail_ok) {
    const T* kt = static_cast<const T*>(p.k_cache) + ((size_t)tail_phys * p.Hkv + h) * p.P * p.D + tc * VEC;
    const uint32_t dst = smem_addr(s_tk + tc * VEC);
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
      const int t = tgrp + k * groups;
      if (t < valid) cp_async16(dst + (uint32_t)(t * p.D * (int)sizeof(T)), kt + (size_t)t * p.D);
    }
    cp_async_commit();
  }
  __syncthreads();
  pdl_wait();                                           // earlier kernels may write the summaries
  // Each warp scores kU pages per round, all of a round's summary rows in
  // flight at once (loading the next round ahead, into a second register
  // set or by cp.async into shared memory, measured slower).
  using Raw = typename RawRow<T, CPL>::type;
  constexpr int kU = sel_unroll<T, CPL>();
  const int span = kSelWarps * kU;
  auto page_ok = [&](int pg) {
    const int ph = s_phys[pg];
    return ph >= 0 && ph < p.num_pages_total;
  };
  auto load = [&](int pg0, Raw (&lo)[kU], Raw (&hi)[kU]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int pg = pg0 + u;
      const int ph = pg < end ? s_phys[pg] : -1;
      if (pg != tail && ph >= 0 && ph < p.num_pages_total) {
        const size_t base = ((size_t)ph * p.Hkv + h) * p.D;
        lo[u] = __ldg(reinterpret_cast<const Raw*>(kmn + base) + lane);
        hi[u] = __ldg(reinterpret_cast<const Raw*>(kmx + base) + lane);
      }
    }
  };
  double wa[CPL], wb[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) { wa[c] = s_ab[0][lane * CPL + c]; wb[c] = s_ab[1][lane * CPL + c]; }
  auto score = [&](int pg0, const Raw (&lo)[kU], const Raw (&hi)[kU]) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int pg = pg0 + u;
      if (pg >= end || pg == tail) continue;              // warp-uniform; the tail page is scored last
      const bool ok = page_ok(pg);
      double acc = 0.0;
      if (ok) {
        float l[CPL], r[CPL];
        RawRow<T, CPL>::unpack(lo[u], l);
        RawRow<T, CPL>::unpack(hi[u], r);
        double acc1 = 0.0;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          acc = fma(wa[c], static_cast<double>(fmaxf(l[c], r[c])), acc);
          acc1 = fma(wb[c], static_cast<double>(fminf(l[c], r[c])), acc1);
        }
        acc += acc1;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        if (!ok) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
        s_keys[pg] = ok ? order_key(acc) : 0ull;
      }
    }
  };
  for (int pg0 = beg + warp * kU; pg0 < end; pg0 += span) {
    Raw lo[kU], hi[kU];
    load(pg0, lo, hi);
    score(pg0, lo, hi);
  }
  // ---- the tail page: min / max over its valid tokens from the staged K
  // (thread = token group x 16-byte chunk of channels; the groups merge by
  // shuffles and across warps), then its score (warp 0)
  if (has_tail) {
    if (tail_ok) {
      cp_async_wait_all();
      __syncthreads();
      float mn[VEC], mx[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) { mn[e] = INFINITY; mx[e] = -INFINITY; }
#pragma unroll
      for (int k = 0; k < kMaxPer; ++k) {
        const int t = tgrp + k * groups;
        if (t >= valid) continue;
        float v[VEC];
        unpack16<T>(*reinterpret_cast<const uint4*>(s_tk + t * p.D + tc * VEC), v);
#pragma unroll
        for (int e = 0; e < VEC; ++e) { mn[e] = fminf(mn[e], v[e]); mx[e] = fmaxf(mx[e], v[e]); }
      }
      for (int o = chunks; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], o));
          mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], o));
        }
      if (lane < chunks)
#pragma unroll
        for (int e = 0; e < VEC; ++e) { s_tpart[0][warp][tc * VEC + e] = mn[e]; s_tpart[1][warp][tc * VEC + e] = mx[e]; }
      __syncthreads();
      if (tid < p.D) {
        float a = INFINITY, z = -INFINITY;
        for (int w = 0; w < kSelWarps; ++w) { a = fminf(a, s_tpart[0][w][tid]); z = fmaxf(z, s_tpart[1][w][tid]); }
        s_tail[0][tid] = a;
        s_tail[1][tid] = z;
      }
      __syncthreads();
    }
    if (warp == 0) {
      double acc = 0.0;
      if (tail_ok) {
        double acc1 = 0.0;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const float l = s_tail[0][lane * CPL + c], r = s_tail[1][lane * CPL + c];
          acc = fma(wa[c], static_cast<double>(fmaxf(l, r)), acc);
          acc1 = fma(wb[c], static_cast<double>(fminf(l, r)), acc1);
        }
        acc += acc1;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        if (!tail_ok) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
        s_keys[tail] = tail_ok ? order_key(acc) : 0ull;
      }
    }
  }
  __syncthreads();
  // ---- copy this CTA's keys into the first CTA (distributed shared memory)
  cluster_wait();                                         // every CTA of the cluster is running
  if (rank != 0) {
    const uint32_t keys_addr = smem_addr(s_keys), phys_addr = smem_addr(s_phys);
    for (int pg = beg + tid; pg < end; pg += kSelThreads) {
      st_cluster_u64(keys_addr + 8u * (uint32_t)pg, 0u, s_keys[pg]);
      st_cluster_u32(phys_addr + 4u * (uint32_t)pg, 0u, s_phys[pg]);
    }
  }
  cluster_sync_all();                                     // all keys are in the first CTA
  if (rank != 0) return;

  // ---- 2. radix select of the budget-th largest key, from the first byte
  // in which the keys differ (all keys share the bits above it)
  unsigned long long kmin_l = ~0ull, kmax_l = 0ull;
  for (int pg = tid; pg < n_b; pg += kSelThreads) {
    const unsigned long long key = s_keys[pg];
    kmin_l = key < kmin_l ? key : kmin_l;
    kmax_l = key > kmax_l ? key : kmax_l;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin_l, o), c = __shfl_xor_sync(0xffffffffu, kmax_l, o);
    kmin_l = a < kmin_l ? a : kmin_l;
    kmax_l = c > kmax_l ? c : kmax_l;
  }
  if (lane == 0) { s_kred[0][warp] = kmin_l; s_kred[1][warp] = kmax_l; }
  __syncthreads();
  if (tid == 0) {
    unsigned long long mn = ~0ull, mx = 0ull;
    for (int w = 0; w < kSelWarps; ++w) {
      mn = s_kred[0][w] < mn ? s_kred[0][w] : mn;
      mx = s_kred[1][w] > mx ? s_kred[1][w] : mx;
    }
    const unsigned long long diff = mn ^ mx;
    const int top = diff ? 8 * ((63 - __clzll((long long)diff)) / 8) : 0;   // highest differing byte
    s_start = top;
    s_shift = 0;                                        // the stop shift, set when a pass ends it
    s_prefix = top >= 56 ? 0ull : (mx >> (top + 8)) << (top + 8);
    s_k = p.budget;
    s_done = 0;
  }
  __syncthreads();
  const int shift0 = s_start;
  for (int shift = shift0; shift >= 0; shift -= 8) {
    s_hist[tid] = 0u;                                      // kSelThreads == 256 bins
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int base = 0; base < n_b; base += kSelThreads) {   // uniform trip count: whole warps
      const int pg = base + tid;
      const unsigned long long key = pg < n_b ? s_keys[pg] : 0ull;
      const bool match = pg < n_b && ((shift >= 56) || (((key ^ prefix) >> (shift + 8)) == 0ull));
      // lanes with the same bin add once (scores often share their top
      // digits); a lane without a match groups only with itself
      const unsigned bin = match ? (unsigned)(key >> shift) & 255u : 256u + (unsigned)lane;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (match && (int)(__ffs(peers) - 1) == lane) atomicAdd(&s_hist[bin], (unsigned)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l, scanned from the top
      unsigned int c[8];
      unsigned int sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = s_hist[255 - 8 * lane - i]; sum += c[i]; }
      unsigned int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int k = s_k;
      const unsigned int excl = incl - sum;
      if (excl < (unsigned)k && incl >= (unsigned)k) {
        unsigned int run = excl;
        for (int i = 0; i < 8; ++i) {
          if (run + c[i] >= (unsigned)k) {
            const unsigned long long digit = 255u - 8u * lane - i;
            s_prefix = prefix | (digit << shift);
            s_k = k - (int)run;
            if (c[i] == (unsigned)(k - (int)run)) { s_done = 1; s_shift = shift; }   // the whole bin is kept
            break;
          }
          run += c[i];
        }
      }
    }
    __syncthreads();
    if (s_done) break;
  }
  const int sh = s_shift;
  const unsigned long long thr = s_prefix >> sh;
  const int need_eq = s_k;

  // ---- 3. compaction in ascending page order (keys compared above the stop digit)
  const int per2 = (n_b + kSelThreads - 1) / kSelThreads;
  const int b0 = min(n_b, tid * per2), b1 = min(n_b, b0 + per2);
  int n_eq = 0;
  for (int pg = b0; pg < b1; ++pg) n_eq += ((s_keys[pg] >> sh) == thr);
  int tot;
  const int eq_before = block_exclusive_scan(n_eq, &tot, s_warp);
  int n_sel = 0;
  {
    int e = eq_before;
    for (int pg = b0; pg < b1; ++pg) {
      const unsigned long long key = s_keys[pg] >> sh;
      if (key > thr) ++n_sel;
      else if (key == thr) { if (e < need_eq) ++n_sel; ++e; }
    }
  }
  int pos = block_exclusive_scan(n_sel, &tot, s_warp);
  {
    int e = eq_before;
    for (int pg = b0; pg < b1; ++pg) {
      const unsigned long long key = s_keys[pg] >> sh;
      bool take = false;
      if (key > thr) take = true;
      else if (key == thr) { take = e < need_eq; ++e; }
      if (take && pos < p.budget) {
        out[pos] = pg;
        out_phys[pos] = s_phys[pg];
        if (pos < kPrefetchPages) prefetch_page(p, s_phys[pg], h);
        ++pos;
      }
    }
  }
}

template <typename T, int CPL, int MINB>
cudaError_t launch_minb(const SelParams& p, int cl, cudaStream_t st) {
  const size_t smem = sel_smem_bytes(p.max_pages, p.P, p.D, (int)sizeof(T));
  cudaError_t e =
      cudaFuncSetAttribute(select_kernel<T, CPL, MINB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(select_kernel<T, CPL, MINB>, dim3(cl, p.Hkv, p.S), dim3(kSelThreads), smem, st, cl, p);
}
template <typename T, int CPL>
cudaError_t launch_typed(const SelParams& p, int cl, bool four, cudaStream_t st) {
  return four ? launch_minb<T, CPL, 4>(p, cl, st) : launch_minb<T, CPL, 2>(p, cl, st);
}

}  // namespace

cudaError_t launch_select(const s3r_paged_kv& kv, const void* kmin, const void* kmax,
                          const void* q, int32_t budget, int32_t* selected, int32_t* selected_phys,
                          uint32_t* status, cudaStream_t st) {
  SelParams p;
  p.q = q;
  p.kmin = kmin;
  p.kmax = kmax;
  p.k_cache = kv.k_cache;
  p.v_cache = kv.v_cache;
  p.block_table = kv.block_table;
  p.context_lens = kv.context_lens;
  p.selected = selected;
  p.selected_phys = selected_phys;
  p.S = kv.num_seqs;
  p.Hq = kv.num_q_heads;
  p.Hkv = kv.num_kv_heads;
  p.G = kv.num_q_heads / kv.num_kv_heads;
  p.D = kv.head_dim;
  p.P = kv.page_size;
  p.max_pages = kv.max_pages_per_seq;
  p.num_pages_total = kv.num_pages_total;
  p.budget = budget;
  p.elt = kv.dtype == S3R_BF16 ? 2 : 4;
  p.status = status;
  // cluster size: the largest of 4, 2, 1 CTAs per (sequence, KV head) such
  // that every CTA of the launch is resident at once, and no more CTAs than
  // 64-page load rounds (larger clusters cannot all be co-scheduled, and a
  // second wave doubles the time). Two CTAs per SM (registers for a round
  // of loads without spills); when the units alone exceed that, the build
  // bounded for four per SM (fewer waves: 299 against 314 us per draft call
  // on the 256-sequence workload; slower where two per SM suffice).
  const long units = (long)kv.num_seqs * kv.num_kv_heads;
  const bool four = units > 2L * device_sm_count();
  const long slots = (four ? 4L : 2L) * device_sm_count();
  int cl = 4;
  while (cl > 1 && (units * cl > slots || (cl - 1) * 64 >= kv.max_pages_per_seq)) cl >>= 1;
  const bool bf = kv.dtype == S3R_BF16;
  cudaError_t e;
  if (kv.head_dim == 128) e = bf ? launch_typed<__nv_bfloat16, 4>(p, cl, four, st) : launch_typed<float, 4>(p, cl, four, st);
  else e = bf ? launch_typed<__nv_bfloat16, 2>(p, cl, four, st) : launch_typed<float, 2>(p, cl, four, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace s3r
