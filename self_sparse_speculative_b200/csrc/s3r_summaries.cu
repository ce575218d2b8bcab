// Per-page key summaries: kmin / kmax over the valid tokens of each page
// (Quest's page metadata; "Quest: Query-Aware Sparsity for Efficient
// Long-Context LLM Inference" on the mlsanity.com page's reference list).
//
// HBM-bound scan: every (page, kv head) tile of P x D keys is read once with
// 16-byte read-only loads; a warp reads whole key rows. Writes are 2 * D
// values per (page, head).
#include <cuda_bf16.h>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kSumThreads = 256;

__device__ __forceinline__ uint4 ldg_nc16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

template <typename T> struct MinMax;

template <> struct MinMax<__nv_bfloat16> {
  __device__ static uint4 lo() { uint32_t x = 0x7F807F80u; return make_uint4(x, x, x, x); }   // +inf
  __device__ static uint4 hi() { uint32_t x = 0xFF80FF80u; return make_uint4(x, x, x, x); }   // -inf
  __device__ static uint32_t mn(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmin2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  __device__ static uint32_t mx(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
};
template <> struct MinMax<float> {
  __device__ static uint4 lo() { uint32_t x = 0x7F800000u; return make_uint4(x, x, x, x); }
  __device__ static uint4 hi() { uint32_t x = 0xFF800000u; return make_uint4(x, x, x, x); }
  __device__ static uint32_t mn(uint32_t a, uint32_t b) { return __float_as_uint(fminf(__uint_as_float(a), __uint_as_float(b))); }
  __device__ static uint32_t mx(uint32_t a, uint32_t b) { return __float_as_uint(fmaxf(__uint_as_float(a), __uint_as_float(b))); }
};

template <typename T>
__device__ __forceinline__ void vmin(uint4& a, const uint4& b) {
  a.x = MinMax<T>::mn(a.x, b.x); a.y = MinMax<T>::mn(a.y, b.y);
  a.z = MinMax<T>::mn(a.z, b.z); a.w = MinMax<T>::mn(a.w, b.w);
}
template <typename T>
__device__ __forceinline__ void vmax(uint4& a, const uint4& b) {
  a.x = MinMax<T>::mx(a.x, b.x); a.y = MinMax<T>::mx(a.y, b.y);
  a.z = MinMax<T>::mx(a.z, b.z); a.w = MinMax<T>::mx(a.w, b.w);
}

struct SumParams {
  const void* k_cache;
  const int32_t* block_table;
  const int32_t* context_lens;
  void* kmin;
  void* kmax;
  int32_t Hkv, D, P, max_pages, num_pages_total;
  int32_t tail_only;
  uint32_t* status;
};

// One CTA per (KV head, page index i, sequence): the P x D tile is split over
// the CTA as (token group, 16-byte channel chunk); every thread reduces its
// few tokens with independent loads, then token groups are merged in shared
// memory. The whole tile is in flight at once, so a tail-page refresh costs
// about one memory latency.
template <typename T>
__global__ void __launch_bounds__(kSumThreads) summaries_kernel(const SumParams p) {
  __shared__ uint4 s_min[kSumThreads];
  __shared__ uint4 s_max[kSumThreads];
  // no early release of the next kernel: the summaries written here are
  // inputs that later calls may read before their grid-dependency wait
  const int h = blockIdx.x, b = blockIdx.z;
  const int L = p.context_lens[b];
  if (L < 1 || L > p.max_pages * p.P) {
    pdl_wait();
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
    return;
  }
  const int n_b = (L + p.P - 1) / p.P;
  const int i = p.tail_only ? n_b - 1 : (int)blockIdx.y;
  if (i >= n_b) {
    pdl_wait();
    return;
  }
  const int phys = p.block_table[(size_t)b * p.max_pages + i];
  if (phys < 0 || phys >= p.num_pages_total) {
    pdl_wait();
    if (threadIdx.x == 0) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
    return;
  }
  const int valid = min(p.P, L - i * p.P);
  constexpr int VEC = 16 / sizeof(T);
  const int chunks = p.D / VEC;                       // 16-byte chunks per key row
  const int groups = kSumThreads / chunks;            // token groups
  const int c = threadIdx.x % chunks, grp = threadIdx.x / chunks;
  const T* base = static_cast<const T*>(p.k_cache) + ((size_t)(phys * p.Hkv + h) * p.P) * p.D + c * VEC;
  uint4 mn = MinMax<T>::lo(), mx = MinMax<T>::hi();
  constexpr int kMaxPer = 8;   // >= 8 token groups x 8 tokens covers P <= 64
  uint4 v[kMaxPer];
#pragma unroll
  for (int k = 0; k < kMaxPer; ++k) {
    const int t = grp + k * groups;
    if (t < valid) v[k] = ldg_nc16(base + (size_t)t * p.D);
  }
#pragma unroll
  for (int k = 0; k < kMaxPer; ++k) {
    const int t = grp + k * groups;
    if (t < valid) { vmin<T>(mn, v[k]); vmax<T>(mx, v[k]); }
  }
  s_min[threadIdx.x] = mn;
  s_max[threadIdx.x] = mx;
  __syncthreads();
  pdl_wait();                                           // earlier kernels may still read the summaries
  if (threadIdx.x < chunks) {
    for (int gi = 1; gi < groups; ++gi) {
      vmin<T>(mn, s_min[gi * chunks + c]);
      vmax<T>(mx, s_max[gi * chunks + c]);
    }
    const size_t o = ((size_t)phys * p.Hkv + h) * p.D + c * VEC;
    *reinterpret_cast<uint4*>(static_cast<T*>(p.kmin) + o) = mn;
    *reinterpret_cast<uint4*>(static_cast<T*>(p.kmax) + o) = mx;
  }
}

}  // namespace

cudaError_t launch_summaries(const s3r_paged_kv& kv, int tail_only, void* kmin, void* kmax,
                             uint32_t* status, cudaStream_t st) {
  SumParams p;
  p.k_cache = kv.k_cache;
  p.block_table = kv.block_table;
  p.context_lens = kv.context_lens;
  p.kmin = kmin;
  p.kmax = kmax;
  p.Hkv = kv.num_kv_heads;
  p.D = kv.head_dim;
  p.P = kv.page_size;
  p.max_pages = kv.max_pages_per_seq;
  p.num_pages_total = kv.num_pages_total;
  p.tail_only = tail_only;
  p.status = status;
  dim3 grid(kv.num_kv_heads, tail_only ? 1 : kv.max_pages_per_seq, kv.num_seqs);
  if (kv.dtype == S3R_BF16)
    return launch_kernel(summaries_kernel<__nv_bfloat16>, grid, dim3(kSumThreads), 0, st, 1, p);
  else
    return launch_kernel(summaries_kernel<float>, grid, dim3(kSumThreads), 0, st, 1, p);
}

}  // namespace s3r
