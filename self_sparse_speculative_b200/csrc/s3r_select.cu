// Query-aware page selection for the sparse draft (Quest-style scoring on
// the mlsanity.com page's reference list; S3R page, Abstract, "uses sparse
// attention to propose tokens").
//
// One CTA per (sequence, KV head):
//   1. score every page p < n_b with the float64 bound
//        s(p) = sum_g sum_d max(q[g,d] * kmin[p,d], q[g,d] * kmax[p,d])
//      over the G query heads of the group, one warp per page (bf16 products
//      are exact in float32; fp32 products are taken in float64);
//   2. radix-select the budget-th largest score on order-preserving 64-bit
//      keys (8 passes of 8 bits: shared-memory histogram, one-warp scan of
//      the 256 bins);
//   3. keep the keys above it plus the lowest-index pages equal to it, and
//      write them in ascending page order with a block-wide prefix sum.
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

__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float load_elem(const float* p, size_t i) { return p[i]; }

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
  const int32_t* block_table;
  const int32_t* context_lens;
  int32_t* selected;        // [S, Hkv, budget]
  int32_t S, Hq, Hkv, G, D, P, max_pages, num_pages_total, budget;
  uint32_t* status;
};

template <typename T>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelParams p) {
  extern __shared__ unsigned long long s_keys[];          // [n_b]
  __shared__ float s_q[8 * 128];                          // [G, D] (bf16 path)
  __shared__ double s_qd[8 * 128];                        // [G, D] (fp32 path)
  __shared__ unsigned int s_hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_k;
  __shared__ int s_warp[kSelWarps];

  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* out = p.selected + ((size_t)b * p.Hkv + h) * p.budget;
  const int L = p.context_lens[b];
  if (L < 1 || L > p.max_pages * p.P) {
    if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
    for (int k = tid; k < p.budget; k += kSelThreads) out[k] = -1;
    return;
  }
  const int n_b = (L + p.P - 1) / p.P;
  if (n_b <= p.budget) {
    for (int k = tid; k < p.budget; k += kSelThreads) out[k] = k < n_b ? k : -1;
    return;
  }

  // ---- 1. scores
  const T* qp = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)h * p.G) * p.D;
  for (int i = tid; i < p.G * p.D; i += kSelThreads) {
    if constexpr (sizeof(T) == 2) s_q[i] = load_elem(qp, i);
    else s_qd[i] = static_cast<double>(load_elem(qp, i));
  }
  __syncthreads();
  const T* kmn = static_cast<const T*>(p.kmin);
  const T* kmx = static_cast<const T*>(p.kmax);
  for (int pg = warp; pg < n_b; pg += kSelWarps) {
    const int phys = p.block_table[(size_t)b * p.max_pages + pg];
    double acc = 0.0;
    const bool ok = phys >= 0 && phys < p.num_pages_total;
    if (ok) {
      const size_t base = ((size_t)phys * p.Hkv + h) * p.D;
      for (int d = lane; d < p.D; d += 32) {
        const float lo = load_elem(kmn, base + d), hi = load_elem(kmx, base + d);
        for (int g = 0; g < p.G; ++g) {
          if constexpr (sizeof(T) == 2) {
            const float qv = s_q[g * p.D + d];
            acc += static_cast<double>(fmaxf(qv * lo, qv * hi));    // bf16 x bf16 is exact in fp32
          } else {
            const double qv = s_qd[g * p.D + d];
            acc += fmax(qv * static_cast<double>(lo), qv * static_cast<double>(hi));
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      if (!ok) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      s_keys[pg] = ok ? order_key(acc) : 0ull;              // a bad page sorts last
    }
  }
  if (tid == 0) { s_prefix = 0ull; s_k = p.budget; }
  __syncthreads();

  // ---- 2. radix select of the budget-th largest key
  for (int shift = 56; shift >= 0; shift -= 8) {
    s_hist[tid] = 0u;                                        // kSelThreads == 256 bins
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int pg = tid; pg < n_b; pg += kSelThreads) {
      const unsigned long long key = s_keys[pg];
      const bool match = (shift == 56) || (((key ^ prefix) >> (shift + 8)) == 0ull);
      if (match) atomicAdd(&s_hist[(key >> shift) & 255u], 1u);
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
        unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int k = s_k;
      const unsigned int excl = incl - sum;
      const bool here = excl < (unsigned)k && incl >= (unsigned)k;
      if (here) {
        unsigned int run = excl;
        for (int i = 0; i < 8; ++i) {
          if (run + c[i] >= (unsigned)k) {
            const unsigned long long digit = 255u - 8u * lane - i;
            s_prefix = prefix | (digit << shift);
            s_k = k - (int)run;
            break;
          }
          run += c[i];
        }
      }
    }
    __syncthreads();
  }
  const unsigned long long thr = s_prefix;
  const int need_eq = s_k;

  // ---- 3. compaction in ascending page order
  const int per = (n_b + kSelThreads - 1) / kSelThreads;
  const int beg = min(n_b, tid * per), end = min(n_b, beg + per);
  int n_eq = 0;
  for (int pg = beg; pg < end; ++pg) n_eq += (s_keys[pg] == thr);
  int tot;
  int eq_before = block_exclusive_scan(n_eq, &tot, s_warp);
  int n_sel = 0;
  {
    int e = eq_before;
    for (int pg = beg; pg < end; ++pg) {
      const unsigned long long key = s_keys[pg];
      if (key > thr) ++n_sel;
      else if (key == thr) { if (e < need_eq) ++n_sel; ++e; }
    }
  }
  int pos = block_exclusive_scan(n_sel, &tot, s_warp);
  {
    int e = eq_before;
    for (int pg = beg; pg < end; ++pg) {
      const unsigned long long key = s_keys[pg];
      bool take = false;
      if (key > thr) take = true;
      else if (key == thr) { take = e < need_eq; ++e; }
      if (take && pos < p.budget) out[pos++] = pg;
    }
  }
}

}  // namespace

cudaError_t launch_select(const s3r_paged_kv& kv, const void* kmin, const void* kmax,
                          const void* q, int32_t budget, int32_t* selected, uint32_t* status,
                          cudaStream_t st) {
  SelParams p;
  p.q = q;
  p.kmin = kmin;
  p.kmax = kmax;
  p.block_table = kv.block_table;
  p.context_lens = kv.context_lens;
  p.selected = selected;
  p.S = kv.num_seqs;
  p.Hq = kv.num_q_heads;
  p.Hkv = kv.num_kv_heads;
  p.G = kv.num_q_heads / kv.num_kv_heads;
  p.D = kv.head_dim;
  p.P = kv.page_size;
  p.max_pages = kv.max_pages_per_seq;
  p.num_pages_total = kv.num_pages_total;
  p.budget = budget;
  p.status = status;
  const size_t smem = (size_t)kv.max_pages_per_seq * sizeof(unsigned long long);
  dim3 grid(kv.num_kv_heads, kv.num_seqs);
  cudaError_t e;
  if (kv.dtype == S3R_BF16) {
    e = cudaFuncSetAttribute(select_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<__nv_bfloat16><<<grid, kSelThreads, smem, st>>>(p);
  } else {
    e = cudaFuncSetAttribute(select_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<float><<<grid, kSelThreads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace s3r
