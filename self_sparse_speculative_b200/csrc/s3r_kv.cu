// KV-cache upkeep of an S3R round ("S3R: Fast and Faithful RL Rollouts via
// Self-Sparse Speculative Decoding", weekinpapers.com, Abstract: the drafter
// and the verifier share the policy's parameters and its KV cache; only the
// accepted drafts and the drawn token are committed).
//
//   kv_append_kernel    rows written at L - overwrite .. L - overwrite + n - 1
//                       (draft steps append one row; verification writes its
//                       R rows over the round's positions), the summaries of
//                       every page holding a written row recomputed over the
//                       page's valid tokens, then L <- L - overwrite + n
//   kv_rollback_kernel  L <- L - R + n_acc + 1 after speculative sampling, the
//                       summary of the new tail page recomputed
//
// One CTA per (KV head, sequence). Every CTA of a sequence reads its length
// before taking a ticket; the last one writes the new length, so the update
// in place never races a reader of the same call. These kernels write inputs
// of later calls (the cache, the summaries, the lengths): they wait for the
// previous kernel before touching anything and never let the next kernel start
// early (no launch_dependents), so the next call sees their writes.
#include <cuda_bf16.h>

#include <cmath>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kKvThreads = 128;

struct KvParams {
  void* k_cache;
  void* v_cache;
  const int32_t* block_table;
  int32_t* lens;
  const void* k_new;          // [S, n, Hkv, D]
  const void* v_new;
  const int32_t* num_accepted;
  void* kmin;
  void* kmax;
  int32_t S, Hkv, D, P, max_pages, num_pages_total;
  int32_t n, overwrite, rows;
  uint32_t* status;
  uint32_t* tickets;          // [S]
};

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }

// kmin / kmax of head h of physical page `phys` over its first `valid` tokens
// (min and max of stored values are exact in the storage type). Each thread
// owns one 16-byte piece of a key row and a token group (tokens tq, tq + ngrp,
// ...), eight rows in flight; the groups merge through shared memory.
template <typename T>
__device__ void summarise_page(const KvParams& p, int phys, int h, int valid) {
  constexpr int kPer = 16 / sizeof(T);
  __shared__ float s_mn[kKvThreads * 8], s_mx[kKvThreads * 8];
  const int pieces = p.D / kPer;                      // 16-byte pieces per row
  const int ngrp = kKvThreads / pieces;
  const int c = threadIdx.x % pieces, tq = threadIdx.x / pieces;
  const T* kt = static_cast<const T*>(p.k_cache) + ((size_t)phys * p.Hkv + h) * p.P * p.D + (size_t)c * kPer;
  float mn[kPer], mx[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) { mn[k] = INFINITY; mx[k] = -INFINITY; }
  for (int t0 = tq; t0 < valid; t0 += 8 * ngrp) {
    uint4 r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = t0 + u * ngrp;
      r[u] = t < valid ? __ldcg(reinterpret_cast<const uint4*>(kt + (size_t)t * p.D)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (t0 + u * ngrp >= valid) break;
      const T* e = reinterpret_cast<const T*>(&r[u]);
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const float v = to_f<T>(e[k]);
        mn[k] = fminf(mn[k], v);
        mx[k] = fmaxf(mx[k], v);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    s_mn[threadIdx.x * kPer + k] = mn[k];
    s_mx[threadIdx.x * kPer + k] = mx[k];
  }
  __syncthreads();
  for (int d = threadIdx.x; d < p.D; d += kKvThreads) {
    const int pc = d / kPer, k = d - (d / kPer) * kPer;
    float a = INFINITY, b = -INFINITY;
    for (int g = 0; g < ngrp; ++g) {
      a = fminf(a, s_mn[(g * pieces + pc) * kPer + k]);
      b = fmaxf(b, s_mx[(g * pieces + pc) * kPer + k]);
    }
    const size_t o = ((size_t)phys * p.Hkv + h) * p.D + d;
    static_cast<T*>(p.kmin)[o] = from_f<T>(a);
    static_cast<T*>(p.kmax)[o] = from_f<T>(b);
  }
  __syncthreads();                                   // the arrays are reused by the next page
}

// The last CTA of sequence b (one per KV head) stores its new length.
__device__ void finish_sequence(const KvParams& p, int b, int new_len, bool write) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.tickets + b, 1u) == (unsigned)(p.Hkv - 1)) {
      if (write) p.lens[b] = new_len;
      p.tickets[b] = 0u;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kKvThreads) kv_append_kernel(const KvParams p) {
  pdl_wait();                                      // earlier kernels may still read the cache
  const int h = blockIdx.x, b = blockIdx.y;
  const int L = __ldcg(p.lens + b);
  const int start = L - p.overwrite, new_len = start + p.n;
  const bool bad = L < 0 || start < 0 || new_len < 1 || new_len > p.max_pages * p.P;
  if (bad) {
    if (threadIdx.x == 0 && h == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
    finish_sequence(p, b, L, false);
    return;
  }
  // the rows, 16-byte pieces (rows are D * sizeof(T) bytes, a multiple of 16)
  constexpr int kPer = 16 / sizeof(T);
  const int pieces = p.D / kPer;
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
  // the keys of the pages to summarise, towards L2 while the rows are copied
  if (p.n > 0)
    for (int pg = start / p.P; pg <= (new_len - 1) / p.P; ++pg) {
      const int phys = bt[pg];
      if (phys < 0 || phys >= p.num_pages_total) continue;
      const char* kp = reinterpret_cast<const char*>(static_cast<const T*>(p.k_cache) +
                                                     ((size_t)phys * p.Hkv + h) * p.P * p.D);
      const int lines = (p.P * p.D * (int)sizeof(T)) / 128;
      for (int l = threadIdx.x; l < lines; l += kKvThreads)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(kp + (size_t)l * 128));
    }
  for (int f = threadIdx.x; f < p.n * pieces; f += kKvThreads) {
    const int t = f / pieces, c = f - (f / pieces) * pieces;
    const int pos = start + t;
    const int phys = bt[pos / p.P];
    if (phys < 0 || phys >= p.num_pages_total) {
      flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
      continue;
    }
    const size_t src = (((size_t)b * p.n + t) * p.Hkv + h) * p.D + (size_t)c * kPer;
    const size_t dst = (((size_t)phys * p.Hkv + h) * p.P + pos % p.P) * p.D + (size_t)c * kPer;
    reinterpret_cast<uint4*>(static_cast<T*>(p.k_cache) + dst)[0] =
        reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + src)[0];
    reinterpret_cast<uint4*>(static_cast<T*>(p.v_cache) + dst)[0] =
        reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + src)[0];
  }
  __syncthreads();                                 // this CTA's rows are visible to its threads
  if (p.n > 0)
    for (int pg = start / p.P; pg <= (new_len - 1) / p.P; ++pg) {
      const int phys = bt[pg];
      if (phys < 0 || phys >= p.num_pages_total) continue;     // flagged above
      summarise_page<T>(p, phys, h, min(p.P, new_len - pg * p.P));
    }
  finish_sequence(p, b, new_len, true);
}

template <typename T>
__global__ void __launch_bounds__(kKvThreads) kv_rollback_kernel(const KvParams p) {
  pdl_wait();
  const int h = blockIdx.x, b = blockIdx.y;
  const int L = __ldcg(p.lens + b);
  const int nacc = __ldcg(p.num_accepted + b);
  const int new_len = L - p.rows + nacc + 1;
  const bool bad = nacc < 0 || nacc >= p.rows || new_len < 1 || L > p.max_pages * p.P;
  if (bad) {
    if (threadIdx.x == 0 && h == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
    finish_sequence(p, b, L, false);
    return;
  }
  const int pg = (new_len - 1) / p.P;
  const int phys = p.block_table[(size_t)b * p.max_pages + pg];
  if (phys < 0 || phys >= p.num_pages_total) {
    if (threadIdx.x == 0) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
  } else {
    summarise_page<T>(p, phys, h, new_len - pg * p.P);
  }
  finish_sequence(p, b, new_len, true);
}

// Launch without programmatic completion: the kernel waits for its
// predecessor (PDL attribute) but its successor starts only when it is done.
template <typename... KArgs, typename... Args>
cudaError_t launch_serial_after(void (*kernel)(KArgs...), dim3 grid, cudaStream_t st, Args... args) {
  return launch_kernel(kernel, grid, dim3(kKvThreads), 0, st, 1, args...);
}

}  // namespace

size_t kv_workspace_bytes(int32_t num_seqs) {
  return align_up(kWsHeader + sizeof(uint32_t) * (size_t)num_seqs, 256);
}

cudaError_t launch_kv_append(const s3r_paged_kv& kv, int32_t* lens, const void* k_new, const void* v_new, int32_t n,
                             int32_t overwrite, void* kmin, void* kmax, void* ws, cudaStream_t st) {
  KvParams p{};
  p.k_cache = const_cast<void*>(kv.k_cache);
  p.v_cache = const_cast<void*>(kv.v_cache);
  p.block_table = kv.block_table;
  p.lens = lens;
  p.k_new = k_new;
  p.v_new = v_new;
  p.kmin = kmin;
  p.kmax = kmax;
  p.S = kv.num_seqs;
  p.Hkv = kv.num_kv_heads;
  p.D = kv.head_dim;
  p.P = kv.page_size;
  p.max_pages = kv.max_pages_per_seq;
  p.num_pages_total = kv.num_pages_total;
  p.n = n;
  p.overwrite = overwrite;
  p.status = static_cast<uint32_t*>(ws);
  p.tickets = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + kWsHeader);
  const dim3 grid(kv.num_kv_heads, kv.num_seqs);
  return kv.dtype == S3R_BF16 ? launch_serial_after(kv_append_kernel<__nv_bfloat16>, grid, st, p)
                              : launch_serial_after(kv_append_kernel<float>, grid, st, p);
}

cudaError_t launch_kv_rollback(const s3r_paged_kv& kv, int32_t* lens, const int32_t* num_accepted, int32_t rows,
                               void* kmin, void* kmax, void* ws, cudaStream_t st) {
  KvParams p{};
  p.k_cache = const_cast<void*>(kv.k_cache);
  p.v_cache = const_cast<void*>(kv.v_cache);
  p.block_table = kv.block_table;
  p.lens = lens;
  p.num_accepted = num_accepted;
  p.kmin = kmin;
  p.kmax = kmax;
  p.S = kv.num_seqs;
  p.Hkv = kv.num_kv_heads;
  p.D = kv.head_dim;
  p.P = kv.page_size;
  p.max_pages = kv.max_pages_per_seq;
  p.num_pages_total = kv.num_pages_total;
  p.rows = rows;
  p.status = static_cast<uint32_t*>(ws);
  p.tickets = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + kWsHeader);
  const dim3 grid(kv.num_kv_heads, kv.num_seqs);
  return kv.dtype == S3R_BF16 ? launch_serial_after(kv_rollback_kernel<__nv_bfloat16>, grid, st, p)
                              : launch_serial_after(kv_rollback_kernel<float>, grid, st, p);
}

}  // namespace s3r
