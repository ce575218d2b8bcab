// Exact speculative sampling of one S3R round, vocab-wide, on the GPU.
//
// S3R page (weekinpapers.com, Abstract): tokens are committed by "exact
// speculative sampling" so that responses follow the dense policy. The rule
// (speculative-sampling papers on the mlsanity.com reference list; restated
// on the ai.info SpecRoll page): accept draft x_i iff u < p_i(x_i)/q_i(x_i);
// at the first rejection j draw from norm(max(p_j - q_j, 0)); if all gamma
// drafts pass, draw a bonus token from p_gamma.
//
// Every kernel works on one vocab chunk per CTA, staged into shared memory
// by a single bulk copy (cp.async.bulk, no multicast) when the rows are
// 16-byte aligned, so a CTA waits for memory once and runs its passes
// on-chip (otherwise it reads global memory directly).
// Pass 1 (one CTA per row chunk): the chunk's max, then the sum of
// exp((x - max)/T) with float32 exponentials into float64. The last CTA of a
// row (atomic ticket) merges the chunk partials into the row's (max, Z); the
// last row of a sequence takes the gamma accept/reject tests (one lane each)
// in float64.
// Pass 2a (residual sequences only): the exact float64 normalisers of the
// two rows the residual is drawn from.
// Pass 2b (one CTA per sequence chunk): float64 draw weights, summed per warp
// segment; the last CTA of a sequence finds, with CTA-wide float64 scans,
// the segment holding u * total and then the token inside it. Every draw is
// decided in float64 on both sides, so it is exact up to the order of the
// float64 sums. float64 exponentials are table-driven (exp_tbl).
// The drafter's own draws (s3r_sample_tokens) are pass 2b alone in "plain"
// mode: one row per draw, weights exp((x - m_c)/T) with m_c the chunk's own
// maximum, brought to the row maximum when the chunks are merged.
// Dependent launches: every kernel releases the next one at its start; pass 1
// and plain draws read their logits (inputs) before the grid-dependency wait,
// so they work while the previous kernel finishes (the wait comes before
// their first workspace write). Released only once every CTA had done its
// chunk instead, the step measured slower on every workload.
#include <cuda_bf16.h>

#include <climits>
#include <cmath>

#include "s3r_device.cuh"
#include "s3r_exp64.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kSmpThreads = 256;
constexpr int kSmpWarps = kSmpThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWarpSegs = kSmpWarps;         // pass-2 chunk = 8 contiguous warp segments
constexpr int kDrawCtasPerSm = 3;            // pass-2 CTAs resident per SM (registers, 72 KB staging)
constexpr int kStatsCtasPerSm = 4;           // pass-1 CTAs resident per SM (registers)
constexpr uint32_t kCopyPiece = 16384;       // bytes per bulk-copy instruction

struct Part1 {
  float m;
  float pad;
  double s;
};

template <typename T> struct LogitIO;
template <> struct LogitIO<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static float at(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
  __device__ static void unpack(const uint4& v, float* x) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};
template <> struct LogitIO<float> {
  static constexpr int kPerVec = 4;
  __device__ static float at(const float* p, size_t i) { return p[i]; }
  __device__ static void unpack(const uint4& v, float* x) {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
  }
};

// n (<= kPerVec) consecutive values at ptr as float: one 16-byte load when
// VEC (ptr 16-byte aligned, in shared or global memory), else scalar loads.
template <typename T, bool VEC>
__device__ __forceinline__ void load_vals(const T* ptr, int n, float* v) {
  using IO = LogitIO<T>;
  if constexpr (VEC) {
    IO::unpack(*reinterpret_cast<const uint4*>(ptr), v);
  } else {
#pragma unroll
    for (int t = 0; t < IO::kPerVec; ++t) v[t] = t < n ? IO::at(ptr, t) : 0.f;
  }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ float block_max(float v, float* s_red) {
  v = warp_max_f(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float r = s_red[0];
  for (int w = 1; w < kSmpWarps; ++w) r = fmaxf(r, s_red[w]);
  __syncthreads();
  return r;
}
__device__ double block_sum_d(double v, double* s_red) {
  v = warp_sum_d(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  double r = 0.0;
  for (int w = 0; w < kSmpWarps; ++w) r += s_red[w];
  __syncthreads();
  return r;
}

// Staging: the CTA's chunk [beg, beg + n) of one or two rows into shared
// memory with bulk copies (thread 0 issues them; every thread waits on the
// mbarrier, which thread 0 initialised before a CTA barrier).
template <typename T>
__device__ void stage_rows(T* s0, const T* g0, T* s1, const T* g1, int n, uint64_t* bar, volatile int* abort,
                           uint32_t* status) {
  const uint32_t bytes = static_cast<uint32_t>(n) * sizeof(T);
  const uint32_t b = smem_addr(bar);
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(b, g1 ? 2u * bytes : bytes);
    for (uint32_t off = 0; off < bytes; off += kCopyPiece) {
      const uint32_t sz = min(kCopyPiece, bytes - off);
      bulk_load(smem_addr(s0) + off, reinterpret_cast<const char*>(g0) + off, sz, b);
      if (g1) bulk_load(smem_addr(s1) + off, reinterpret_cast<const char*>(g1) + off, sz, b);
    }
  }
  mbar_wait(b, 0, abort, status);
}
__device__ __forceinline__ void init_stage_bar(uint64_t* bar) {
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
}

// Row pointers of the spec layout: rows 0..R-1 target, R..2*gamma draft.
template <typename T>
__device__ __forceinline__ const T* row_ptr(const SampleParams& p, bool spec, int row) {
  if (!spec) return static_cast<const T*>(p.target) + (size_t)row * p.vocab;
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  const int b = row / per, rr = row - (row / per) * per;
  if (rr < R) return static_cast<const T*>(p.target) + ((size_t)b * R + rr) * p.vocab;
  return static_cast<const T*>(p.draft) + ((size_t)b * p.gamma + (rr - R)) * p.vocab;
}

// Accept/reject tests of sequence b, one lane per draft position (warp 0).
template <typename T>
__device__ void decide(const SampleParams& p, int b) {
  const int lane = threadIdx.x & 31;
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  bool acc = true;
  int x = 0;
  if (lane < p.gamma) {
    x = p.draft_tokens[(size_t)b * p.gamma + lane];
    double ratio = 0.0;
    if (x >= 0 && x < p.vocab) {
      // statistics written by other CTAs of this grid: read through L2
      const double* st = p.stats + 2 * ((size_t)b * per + lane);
      const double* sd = p.draft_stats ? p.draft_stats + 2 * ((size_t)b * p.gamma + lane)
                                       : p.stats + 2 * ((size_t)b * per + R + lane);
      const double lt = LogitIO<T>::at(static_cast<const T*>(p.target) + ((size_t)b * R + lane) * p.vocab, x);
      const double ld = LogitIO<T>::at(static_cast<const T*>(p.draft) + ((size_t)b * p.gamma + lane) * p.vocab, x);
      const double px = exp((lt - __ldcg(st)) * p.inv_temp_d) / __ldcg(st + 1);
      const double qx = exp((ld - __ldcg(sd)) * p.inv_temp_d) / __ldcg(sd + 1);
      ratio = qx > 0.0 ? px / qx : 0.0;
    } else {
      flag_status(p.status, S3R_DEV_BAD_TOKEN_ID);
    }
    acc = static_cast<double>(p.u_accept[(size_t)b * p.gamma + lane]) < ratio;
  }
  const unsigned rej = __ballot_sync(0xffffffffu, !acc) & ((1u << p.gamma) - 1u);
  const int j = rej ? __ffs(rej) - 1 : p.gamma;         // first rejected position
  for (int i = lane; i < R; i += 32) {
    if (i < j) p.out_tokens[(size_t)b * R + i] = p.draft_tokens[(size_t)b * p.gamma + i];
    else if (i > j) p.out_tokens[(size_t)b * R + i] = -1;
  }
  if (lane == 0) {
    p.num_accepted[b] = j;
    p.jsel[b] = j;
  }
}

// ---------------------------------------------------------------- pass 1
// One streaming pass per chunk: every thread keeps a running maximum m and
// the float32 sum of 2^((x - m) log2(e)/T), rescaled when m grows (the
// online normaliser of M. Milakov and N. Gimelshein, "Online normalizer
// calculation for softmax", 2018); four 16-byte loads in flight per thread.
// VEC: rows 16-byte aligned with a length that is a multiple of the vector.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kSmpThreads, kStatsCtasPerSm) rowstats_kernel(const SampleParams p) {
  pdl_launch_dependents();
  __shared__ float s_redf[kSmpWarps];
  __shared__ double s_redd[kSmpWarps];
  __shared__ int s_last;
  using IO = LogitIO<T>;
  constexpr int PV = IO::kPerVec;
  constexpr int kB = 4;                                 // vectors in flight per thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  // with the draft rows' statistics given, only the target rows are visited
  const int tr = blockIdx.x / p.c1, c = blockIdx.x - (blockIdx.x / p.c1) * p.c1;
  const int row = p.draft_stats ? (tr / R) * per + (tr - (tr / R) * R) : tr;
  const int rows_per_seq = p.draft_stats ? R : per;
  const int beg = c * p.ch1, n = min(p.vocab, beg + p.ch1) - beg;
  const T* src = row_ptr<T>(p, true, row) + beg;
  const float k2 = kLog2e * p.inv_temp;
  float m = -INFINITY, nmk = INFINITY;                  // nmk = -m k2
  double s = 0.0;
  for (int i0 = tid * PV; i0 < n; i0 += kB * kSmpThreads * PV) {
    float v[kB][PV];
    int cnt[kB];
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int i = i0 + b * kSmpThreads * PV;
      cnt[b] = max(0, min(PV, n - i));
      if (cnt[b] > 0) load_vals<T, VEC>(src + i, cnt[b], v[b]);
    }
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      if (cnt[b] <= 0) continue;
      const bool full = VEC || cnt[b] == PV;            // VEC: whole vectors only
      float vm = -INFINITY;
#pragma unroll
      for (int t = 0; t < PV; ++t)
        if (full || t < cnt[b]) vm = fmaxf(vm, v[b][t]);
      if (vm > m) {
        s *= static_cast<double>(ex2((m - vm) * k2));   // from m = -inf: a factor 0 on s = 0
        m = vm;
        nmk = -m * k2;
      }
      if (m == -INFINITY) continue;                     // nothing but -inf so far
      // a vector's exponentials summed pairwise in float32, then added in float64
      float e[PV];
#pragma unroll
      for (int t = 0; t < PV; ++t) e[t] = (full || t < cnt[b]) ? ex2(fmaf(v[b][t], k2, nmk)) : 0.f;
#pragma unroll
      for (int w = PV / 2; w > 0; w >>= 1)
#pragma unroll
        for (int t = 0; t < w; ++t) e[t] += e[t + w];
      s += static_cast<double>(e[0]);
    }
  }
  const float M = block_max(m, s_redf);
  const double sc = m == -INFINITY ? 0.0 : s * static_cast<double>(ex2((m - M) * k2));
  const double S = block_sum_d(sc, s_redd);
  // the logits are inputs: only the workspace waits for the previous kernel
  pdl_wait();
  if (tid == 0) {
    Part1* part = static_cast<Part1*>(p.part1) + (size_t)row * p.c1 + c;
    part->m = M;
    part->s = S;
    __threadfence();
    s_last = (atomicAdd(p.tk_row + row, 1u) == (unsigned)(p.c1 - 1));
  }
  __syncthreads();
  if (!s_last || warp != 0) return;
  // last CTA of the row: merge chunk partials in float64 (warp 0)
  __threadfence();
  const Part1* part = static_cast<const Part1*>(p.part1) + (size_t)row * p.c1;
  float Mr = -INFINITY;
  for (int i = lane; i < p.c1; i += 32) Mr = fmaxf(Mr, __ldcg(&part[i].m));
  Mr = warp_max_f(Mr);
  double Z = 0.0;
  for (int i = lane; i < p.c1; i += 32) {
    const float mi = __ldcg(&part[i].m);
    if (mi != -INFINITY)
      Z += __ldcg(&part[i].s) * exp((static_cast<double>(mi) - static_cast<double>(Mr)) * p.inv_temp_d);
  }
  Z = warp_sum_d(Z);
  if (lane == 0) {
    p.stats[2 * (size_t)row] = Mr;
    p.stats[2 * (size_t)row + 1] = Z;
    p.tk_row[row] = 0u;
  }
  const int b = row / per;
  int last = 0;
  if (lane == 0) {
    __threadfence();
    last = atomicAdd(p.tk_seq1 + b, 1u) == (unsigned)(rows_per_seq - 1);
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) {
    __threadfence();
    if (lane == 0) p.tk_seq1[b] = 0u;
    decide<T>(p, b);
  }
}

// ---------------------------------------------------------------- pass 2
// The rows and normalisers a draw uses.
struct DrawRows {
  const void* prow;      // p row (target j, target gamma, or the plain row)
  const void* qrow;      // residual: draft row j, else null
  double Mp, Mq;         // row maxima (shifts)
  double iZp, iZq;       // residual: exact 1/Z of the two rows; else 1
};

template <typename T, bool SPEC>
__device__ DrawRows draw_rows(const SampleParams& p, int s, int j) {
  DrawRows w;
  w.iZp = 1.0;
  w.iZq = 1.0;
  w.qrow = nullptr;
  w.Mq = 0.0;
  if (!SPEC) {                                          // the shift is the chunk's own maximum
    w.prow = static_cast<const T*>(p.target) + (size_t)s * p.vocab;
    w.Mp = 0.0;
    return w;
  }
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  w.prow = static_cast<const T*>(p.target) + ((size_t)s * R + j) * p.vocab;
  w.Mp = p.stats[2 * ((size_t)s * per + j)];
  if (j < p.gamma) {
    w.qrow = static_cast<const T*>(p.draft) + ((size_t)s * p.gamma + j) * p.vocab;
    w.Mq = p.draft_stats ? p.draft_stats[2 * ((size_t)s * p.gamma + j)] : p.stats[2 * ((size_t)s * per + R + j)];
    w.iZp = 1.0 / __ldcg(p.znorm + 2 * (size_t)s);
    w.iZq = 1.0 / __ldcg(p.znorm + 2 * (size_t)s + 1);
  }
  return w;
}

// float64 draw weights of the n (<= kPerVec) elements at pa (and pb for a
// residual): exp((a - Mp)/T) iZp, or max(that - exp((b - Mq)/T) iZq, 0).
// G: elements whose exponentials are interleaved (fewer for two rows, to
// bound the registers).
template <typename T, bool VEC, int G = 4>
__device__ __forceinline__ void weights(const DrawRows& w, const T* pa, const T* pb, int n, double invT,
                                        const double* tab, double* out) {
  using IO = LogitIO<T>;
  constexpr int PV = IO::kPerVec;
  float a[PV], b[PV];
  load_vals<T, VEC>(pa, n, a);
  if (w.qrow) load_vals<T, VEC>(pb, n, b);
  const double ca = -w.Mp * invT, cb = -w.Mq * invT;    // (x - M)/T as one fused multiply-add
  // Every argument is <= 0 (shift = a maximum), so exp_tbl needs its fix-up
  // only below -707: decided once per vector from its smallest value. VEC
  // vectors are whole (n == PV).
  float amin = a[0], bmin = w.qrow ? b[0] : 0.f;
#pragma unroll
  for (int t = 1; t < PV; ++t)
    if (VEC || t < n) {
      amin = fminf(amin, a[t]);
      if (w.qrow) bmin = fminf(bmin, b[t]);
    }
  const bool in_range = fma(static_cast<double>(amin), invT, ca) > -707.0 &&
                        (!w.qrow || fma(static_cast<double>(bmin), invT, cb) > -707.0);
#pragma unroll
  for (int t0 = 0; t0 < PV; t0 += G) {
    double xa[G], xb[G], ea[G], eb[G];
#pragma unroll
    for (int t = 0; t < G; ++t) {                       // branch-free
      xa[t] = fma(static_cast<double>(a[t0 + t]), invT, ca);
      ea[t] = exp_tbl(xa[t], tab);
      if (w.qrow) {
        xb[t] = fma(static_cast<double>(b[t0 + t]), invT, cb);
        eb[t] = exp_tbl(xb[t], tab);
      }
    }
    if (!in_range) {
#pragma unroll
      for (int t = 0; t < G; ++t) {
        ea[t] = exp_fixup(xa[t], ea[t], tab);
        if (w.qrow) eb[t] = exp_fixup(xb[t], eb[t], tab);
      }
    }
#pragma unroll
    for (int t = 0; t < G; ++t) {
      const double pe = ea[t] * w.iZp;
      double wt = pe;
      if (w.qrow) {
        const double qe = eb[t] * w.iZq;
        wt = pe > qe ? pe - qe : 0.0;
      }
      out[t0 + t] = (VEC || t0 + t < n) ? wt : 0.0;
    }
  }
}
template <typename T, bool VEC>
__device__ __forceinline__ void weights_at(const DrawRows& w, int e, int n, double invT, const double* tab,
                                           double* out) {
  weights<T, VEC, 2>(w, static_cast<const T*>(w.prow) + e, w.qrow ? static_cast<const T*>(w.qrow) + e : nullptr, n,
                  invT, tab, out);
}

// Pass 2a: exact float64 normalisers of the residual's two rows.
template <typename T, bool STAGE>
__global__ void __launch_bounds__(kSmpThreads, kDrawCtasPerSm) znorm_kernel(const SampleParams p) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t s_dyn[];
  __shared__ uint64_t s_bar;
  __shared__ int s_abort;
  __shared__ double s_red[2][kSmpWarps];
  __shared__ double s_tab[kExpTab];
  __shared__ int s_last;
  using IO = LogitIO<T>;
  constexpr int PV = IO::kPerVec;
  const int s = blockIdx.x / p.c2, c = blockIdx.x - (blockIdx.x / p.c2) * p.c2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = p.jsel[s];
  if (j >= p.gamma) return;                              // bonus draw: no residual (uniform per sequence)
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  // with the draft rows' statistics given, the draft row's exact Z is known:
  // only the target row is summed here
  const bool two = p.draft_stats == nullptr;
  const double Mp = p.stats[2 * ((size_t)s * per + j)];
  const double Mq = two ? p.stats[2 * ((size_t)s * per + R + j)] : 0.0;
  const int beg = c * p.ch2, n = min(p.vocab, beg + p.ch2) - beg;
  const T* pa = static_cast<const T*>(p.target) + ((size_t)s * R + j) * p.vocab + beg;
  const T* pb = static_cast<const T*>(p.draft) + ((size_t)s * p.gamma + j) * p.vocab + beg;
  fill_exp_tab(s_tab);
  if constexpr (STAGE) {
    if (tid == 0) s_abort = 0;
    init_stage_bar(&s_bar);
    T* s0 = reinterpret_cast<T*>(s_dyn);
    T* s1 = s0 + p.ch2;
    stage_rows<T>(s0, pa, two ? s1 : nullptr, two ? pb : nullptr, n, &s_bar, &s_abort, p.status);
    pa = s0;
    pb = s1;
  } else {
    __syncthreads();
  }
  double zt = 0.0, zd = 0.0;
  if (!two) {
    // the target row alone
    const double ca = -Mp * p.inv_temp_d;
    for (int i = tid * PV; i < n; i += kSmpThreads * PV) {
      const int m = min(PV, n - i);
      float a[PV];
      load_vals<T, STAGE>(pa + i, m, a);
      float amin = a[0];
#pragma unroll
      for (int t = 1; t < PV; ++t)
        if (STAGE || t < m) amin = fminf(amin, a[t]);
      const bool in_range = fma(static_cast<double>(amin), p.inv_temp_d, ca) > -707.0;
#pragma unroll
      for (int t0 = 0; t0 < PV; t0 += 4) {
        double xa[4], ea[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          xa[t] = fma(static_cast<double>(a[t0 + t]), p.inv_temp_d, ca);
          ea[t] = exp_tbl(xa[t], s_tab);
        }
        if (!in_range)
#pragma unroll
          for (int t = 0; t < 4; ++t) ea[t] = exp_fixup(xa[t], ea[t], s_tab);
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (STAGE || t0 + t < m) zt += ea[t];
      }
    }
  }
  const double ca = -Mp * p.inv_temp_d, cb = -Mq * p.inv_temp_d;
  for (int i = tid * PV; two && i < n; i += kSmpThreads * PV) {
    const int m = min(PV, n - i);
    float a[PV], b[PV];
    load_vals<T, STAGE>(pa + i, m, a);
    load_vals<T, STAGE>(pb + i, m, b);
    // arguments are <= 0: the exp_tbl fix-up only below -707, decided per
    // vector (staged vectors are whole)
    float amin = a[0], bmin = b[0];
#pragma unroll
    for (int t = 1; t < PV; ++t)
      if (STAGE || t < m) {
        amin = fminf(amin, a[t]);
        bmin = fminf(bmin, b[t]);
      }
    const bool in_range = fma(static_cast<double>(amin), p.inv_temp_d, ca) > -707.0 &&
                          fma(static_cast<double>(bmin), p.inv_temp_d, cb) > -707.0;
#pragma unroll
    for (int t0 = 0; t0 < PV; t0 += 4) {
      double xa[4], xb[4], ea[4], eb[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {                     // branch-free
        xa[t] = fma(static_cast<double>(a[t0 + t]), p.inv_temp_d, ca);
        xb[t] = fma(static_cast<double>(b[t0 + t]), p.inv_temp_d, cb);
        ea[t] = exp_tbl(xa[t], s_tab);
        eb[t] = exp_tbl(xb[t], s_tab);
      }
      if (!in_range) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          ea[t] = exp_fixup(xa[t], ea[t], s_tab);
          eb[t] = exp_fixup(xb[t], eb[t], s_tab);
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (STAGE || t0 + t < m) {
          zt += ea[t];
          zd += eb[t];
        }
      }
    }
  }
  zt = warp_sum_d(zt);
  zd = warp_sum_d(zd);
  if (lane == 0) { s_red[0][warp] = zt; s_red[1][warp] = zd; }
  __syncthreads();
  if (tid == 0) {
    double a = 0.0, b = 0.0;
    for (int i = 0; i < kSmpWarps; ++i) { a += s_red[0][i]; b += s_red[1][i]; }
    p.zpart[2 * ((size_t)s * p.c2 + c)] = a;
    p.zpart[2 * ((size_t)s * p.c2 + c) + 1] = b;
    __threadfence();
    s_last = atomicAdd(p.tk_seq3 + s, 1u) == (unsigned)(p.c2 - 1);
  }
  __syncthreads();
  if (!s_last || warp != 0) return;
  __threadfence();
  double a = 0.0, b = 0.0;
  for (int i = lane; i < p.c2; i += 32) {
    a += __ldcg(p.zpart + 2 * ((size_t)s * p.c2 + i));
    b += __ldcg(p.zpart + 2 * ((size_t)s * p.c2 + i) + 1);
  }
  a = warp_sum_d(a);
  b = warp_sum_d(b);
  if (lane == 0) {
    p.znorm[2 * (size_t)s] = a;
    p.znorm[2 * (size_t)s + 1] = two ? b : p.draft_stats[2 * ((size_t)s * p.gamma + j) + 1];
    p.tk_seq3[s] = 0u;
  }
}

// Inclusive scan of one float64 per thread over the CTA; *total gets the CTA
// total. Every thread calls it; it ends with the CTA synchronised.
__device__ double block_scan_d(double v, double* total, double* s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_w[warp] = x;
  __syncthreads();
  double off = 0.0, tot = 0.0;
#pragma unroll
  for (int w = 0; w < kSmpWarps; ++w) {
    const double sw = s_w[w];
    if (w < warp) off += sw;
    tot += sw;
  }
  __syncthreads();
  *total = tot;
  return x + off;
}

// Thread t's contiguous share [e0, e1) of [b0, b1), aligned to the vector width.
template <int PV>
__device__ __forceinline__ void thread_range(int b0, int b1, int* e0, int* e1) {
  int E = (b1 - b0 + kSmpThreads - 1) / kSmpThreads;
  E = (E + PV - 1) / PV * PV;
  *e0 = min(b1, b0 + (int)threadIdx.x * E);
  *e1 = min(b1, *e0 + E);
}

// Sum of the draw weights over [b0, b1) (every thread calls it).
template <typename T, bool VEC>
__device__ double block_total(const DrawRows& w, int b0, int b1, double invT, const double* tab, double* s_w) {
  constexpr int PV = LogitIO<T>::kPerVec;
  int e0, e1;
  thread_range<PV>(b0, b1, &e0, &e1);
  double loc = 0.0;
  for (int e = e0; e < e1; e += PV) {
    double wv[PV];
    weights_at<T, VEC>(w, e, min(PV, e1 - e), invT, tab, wv);
#pragma unroll
    for (int t = 0; t < PV; ++t) loc += wv[t];
  }
  double tot;
  block_scan_d(loc, &tot, s_w);
  return tot;
}

// The first k in [b0, b1) whose running sum (from `base`) exceeds thr, found
// by the whole CTA: every thread sums its share, a block scan gives each
// share's starting sum, and the one thread whose share crosses thr walks it.
// Without a crossing (rounding) the last index with positive weight is
// returned (-1 if none). Every thread calls it and gets the same k.
template <typename T, bool VEC>
__device__ int block_find(const DrawRows& w, int b0, int b1, double base, double thr, double invT,
                          const double* tab, double* s_w, int* s_i) {
  constexpr int PV = LogitIO<T>::kPerVec;
  int e0, e1;
  thread_range<PV>(b0, b1, &e0, &e1);
  if (threadIdx.x == 0) { s_i[0] = INT_MAX; s_i[1] = -1; s_i[2] = -1; }
  double loc = 0.0;
  int lastpos = -1;
  for (int e = e0; e < e1; e += PV) {
    double wv[PV];
    weights_at<T, VEC>(w, e, min(PV, e1 - e), invT, tab, wv);
#pragma unroll
    for (int t = 0; t < PV; ++t) {
      loc += wv[t];
      if (wv[t] > 0.0) lastpos = e + t;
    }
  }
  double tot;
  const double incl = block_scan_d(loc, &tot, s_w);        // also orders the s_i initialisation
  const double before = base + (incl - loc);
  if (loc > 0.0 && before + loc > thr) atomicMin(&s_i[0], (int)threadIdx.x);
  if (lastpos >= 0) atomicMax(&s_i[1], lastpos);
  __syncthreads();
  const int winner = s_i[0];
  int k;
  if (winner != INT_MAX) {
    if ((int)threadIdx.x == winner) {
      double run = before;
      int kk = -1, lp = -1;
      for (int e = e0; e < e1 && kk < 0; e += PV) {
        double wv[PV];
        weights_at<T, VEC>(w, e, min(PV, e1 - e), invT, tab, wv);
#pragma unroll
        for (int t = 0; t < PV; ++t) {
          run += wv[t];
          if (wv[t] > 0.0) lp = e + t;
          if (kk < 0 && run > thr) kk = e + t;
        }
      }
      s_i[2] = kk >= 0 ? kk : lp;
    }
    __syncthreads();
    k = s_i[2];
  } else {
    k = s_i[1];
  }
  __syncthreads();
  return k;
}

// Pass 2b: the draw. Spec draws shift by the row statistics of pass 1; plain
// draws (the drafter's own) shift every chunk by its own maximum and bring
// the chunk sums to the row maximum with an exact float64 factor when the
// chunks are merged, so they need no statistics pass.
template <typename T, bool SPEC, bool STAGE>
__global__ void __launch_bounds__(kSmpThreads, kDrawCtasPerSm) draw_kernel(const SampleParams p) {
  pdl_launch_dependents();
  // speculative draws start from the earlier passes' results; plain draws
  // read only inputs (the logits) until their first workspace write
  if constexpr (SPEC) pdl_wait();
  extern __shared__ __align__(16) uint8_t s_dyn[];
  __shared__ uint64_t s_bar;
  __shared__ int s_abort;
  __shared__ double s_w[kSmpWarps];
  __shared__ double s_tab[kExpTab];
  __shared__ float s_redf[kSmpWarps];
  __shared__ int s_i[3];
  __shared__ double s_base;
  __shared__ int s_last;
  using IO = LogitIO<T>;
  constexpr int PV = IO::kPerVec;
  const int s = blockIdx.x / p.c2, c = blockIdx.x - (blockIdx.x / p.c2) * p.c2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  fill_exp_tab(s_tab);
  const int j = SPEC ? p.jsel[s] : 0;
  DrawRows w = draw_rows<T, SPEC>(p, s, j);
  const int cbeg = c * p.ch2, n = min(p.vocab, cbeg + p.ch2) - cbeg;
  const T* ca = static_cast<const T*>(w.prow) + cbeg;   // this chunk of the rows
  const T* cb = w.qrow ? static_cast<const T*>(w.qrow) + cbeg : nullptr;
  if constexpr (STAGE) {
    if (tid == 0) s_abort = 0;
    init_stage_bar(&s_bar);                              // also orders the exp table
    T* s0 = reinterpret_cast<T*>(s_dyn);
    T* s1 = w.qrow ? s0 + p.ch2 : nullptr;
    stage_rows<T>(s0, ca, s1, cb, n, &s_bar, &s_abort, p.status);
    ca = s0;
    cb = s1;
  }
  const int seg = p.ch2 / kWarpSegs;                     // elements per warp segment
  const int sb0 = min(n, warp * seg), sb1 = min(n, sb0 + seg);
  float* cmax = p.cmax + (size_t)s * p.c2;
  float Mc = -INFINITY;
  if constexpr (!SPEC) {
    float mx = -INFINITY;
    for (int i = sb0 + lane * PV; i < sb1; i += 32 * PV) {
      float v[PV];
      const int m = min(PV, sb1 - i);
      load_vals<T, STAGE>(ca + i, m, v);
#pragma unroll
      for (int t = 0; t < PV; ++t)
        if (t < m) mx = fmaxf(mx, v[t]);
    }
    Mc = block_max(mx, s_redf);                          // synchronises (orders the exp table too)
    w.Mp = Mc == -INFINITY ? 0.0 : static_cast<double>(Mc);
  } else {
    __syncthreads();
  }
  double acc = 0.0;
  for (int i = sb0 + lane * PV; i < sb1; i += 32 * PV) {
    double wv[PV];
    weights<T, STAGE, SPEC ? 2 : 4>(w, ca + i, cb ? cb + i : nullptr, min(PV, sb1 - i), p.inv_temp_d, s_tab, wv);
#pragma unroll
    for (int t = 0; t < PV; ++t) acc += wv[t];
  }
  acc = warp_sum_d(acc);
  if constexpr (!SPEC) {
    pdl_wait();                                          // outputs and the workspace from here on
    if (tid == 0) cmax[c] = Mc;
  }
  if (lane == 0) {
    p.wpart[((size_t)s * p.c2 + c) * kWarpSegs + warp] = acc;
    __threadfence();
  }
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.tk_seq2 + s, 1u) == (unsigned)(p.c2 - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- last CTA of the sequence (all threads): the draw
  const int R = p.gamma + 1;
  const double u = SPEC ? static_cast<double>(p.u_sample[(size_t)s * R + j]) : static_cast<double>(p.u_sample[s]);
  const double* wp = p.wpart + (size_t)s * p.c2 * kWarpSegs;
  const int nseg = p.c2 * kWarpSegs;
  double Mrow = 0.0;
  if constexpr (!SPEC) {
    float m = -INFINITY;
    for (int i = tid; i < p.c2; i += kSmpThreads) m = fmaxf(m, __ldcg(cmax + i));
    Mrow = static_cast<double>(block_max(m, s_redf));
  }
  // chunk c's factor to the row shift (plain draws), 1 for spec draws
  auto chunk_scale = [&](int cc, float* mc_out) -> double {
    if constexpr (SPEC) {
      *mc_out = 0.f;
      return 1.0;
    } else {
      const float mc = __ldcg(cmax + cc);
      *mc_out = mc;
      if (mc == -INFINITY) return 0.0;
      const double x = (static_cast<double>(mc) - Mrow) * p.inv_temp_d;
      return exp_fixup(x, exp_tbl(x, s_tab), s_tab);
    }
  };
  auto segval = [&](int i) -> double {
    const double v = __ldcg(wp + i);
    if constexpr (SPEC) return v;
    float mc;
    return v == 0.0 ? 0.0 : v * chunk_scale(i / kWarpSegs, &mc);
  };
  double loc = 0.0;
  for (int i = tid; i < nseg; i += kSmpThreads) loc += segval(i);
  double total;
  block_scan_d(loc, &total, s_w);
  if constexpr (!SPEC) {
    // the row's statistics at temperature T: its largest logit and the exact
    // float64 sum of exp((x - max) / T) (the chunk sums brought to the row max)
    if (p.row_stats_out && tid == 0) {
      p.row_stats_out[2 * (size_t)s] = Mrow;
      p.row_stats_out[2 * (size_t)s + 1] = total;
    }
  }
  int k = -1;
  if (total > 0.0) {
    const double thr = u * total;
    // the first segment whose running sum passes thr (rounds of one segment per thread)
    if (tid == 0) { s_i[0] = INT_MAX; s_i[1] = -1; }
    double carry = 0.0;
    for (int i0 = 0; i0 < nseg; i0 += kSmpThreads) {
      const int i = i0 + tid;
      const double v = i < nseg ? segval(i) : 0.0;
      double rt;
      const double incl = carry + block_scan_d(v, &rt, s_w);
      if (v > 0.0) {
        atomicMax(&s_i[1], i);
        if (incl > thr) atomicMin(&s_i[0], i);
      }
      __syncthreads();
      if (i == s_i[0]) s_base = incl - v;
      __syncthreads();
      if (s_i[0] != INT_MAX) break;
      carry += rt;
    }
    int sel = s_i[0];
    double base;
    if (sel != INT_MAX) {
      base = s_base;
    } else {                                             // rounding left no crossing: last segment with weight
      sel = s_i[1];
      double l2 = 0.0;
      for (int i = tid; i < sel; i += kSmpThreads) l2 += segval(i);
      block_scan_d(l2, &base, s_w);
    }
    __syncthreads();
    if (sel >= 0) {
      const int cc = sel / kWarpSegs, ww = sel - cc * kWarpSegs;
      const int b0 = min(p.vocab, cc * p.ch2 + ww * seg), b1 = min(min(p.vocab, cc * p.ch2 + p.ch2), b0 + seg);
      DrawRows ws = w;
      if constexpr (!SPEC) {
        float mc;
        ws.iZp = chunk_scale(cc, &mc);
        ws.Mp = mc == -INFINITY ? 0.0 : static_cast<double>(mc);
      }
      k = block_find<T, STAGE>(ws, b0, b1, base, thr, p.inv_temp_d, s_tab, s_w, s_i);
    }
  } else if (SPEC && w.qrow) {
    // all-zero residual (p_j == q_j after rounding): draw from p_j instead
    DrawRows wb = w;
    wb.qrow = nullptr;
    wb.iZp = 1.0;
    const double tot = block_total<T, STAGE>(wb, 0, p.vocab, p.inv_temp_d, s_tab, s_w);
    k = block_find<T, STAGE>(wb, 0, p.vocab, 0.0, u * tot, p.inv_temp_d, s_tab, s_w, s_i);
  }
  if (tid == 0) {
    if (k < 0) k = 0;
    if (SPEC) p.out_tokens[(size_t)s * R + j] = k;
    else p.out_tokens[s] = k;
    p.tk_seq2[s] = 0u;
  }
}

template <typename T, bool SPEC>
cudaError_t launch_typed(const SampleParams& p, cudaStream_t st) {
  const int per = SPEC ? 2 * p.gamma + 1 : 1;
  const int nrows = p.nseq * (SPEC && p.draft_stats ? p.gamma + 1 : per);   // rows of the statistics pass
  // bulk staging needs 16-byte aligned rows
  const bool stage = (((size_t)p.vocab * sizeof(T)) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(p.target) % 16 == 0) &&
                     (!SPEC || reinterpret_cast<uintptr_t>(p.draft) % 16 == 0);
  const dim3 blk(kSmpThreads);
  const size_t sm2 = stage ? (size_t)p.ch2 * sizeof(T) * (SPEC ? 2 : 1) : 0;
  cudaError_t e = cudaSuccess;
  if (SPEC) {
    if (stage) e = launch_kernel(rowstats_kernel<T, true>, dim3(p.c1 * nrows), blk, 0, st, 1, p);
    else e = launch_kernel(rowstats_kernel<T, false>, dim3(p.c1 * nrows), blk, 0, st, 1, p);
    if (e != cudaSuccess) return e;
    if (stage) {
      e = cudaFuncSetAttribute(znorm_kernel<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
      if (e == cudaSuccess) e = launch_kernel(znorm_kernel<T, true>, dim3(p.c2 * p.nseq), blk, sm2, st, 1, p);
    } else {
      e = launch_kernel(znorm_kernel<T, false>, dim3(p.c2 * p.nseq), blk, 0, st, 1, p);
    }
    if (e != cudaSuccess) return e;
  }
  if (stage) {
    e = cudaFuncSetAttribute(draw_kernel<T, SPEC, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    if (e != cudaSuccess) return e;
    return launch_kernel(draw_kernel<T, SPEC, true>, dim3(p.c2 * p.nseq), blk, sm2, st, 1, p);
  }
  return launch_kernel(draw_kernel<T, SPEC, false>, dim3(p.c2 * p.nseq), blk, 0, st, 1, p);
}

// Diagnostic: the sampler's float64 exponential (exp_tbl with exp_fixup, as
// the draw kernels evaluate it) and CUDA's exp() of the same arguments.
__global__ void __launch_bounds__(kSmpThreads) exp64_probe_kernel(const double* x, double* y_tbl, double* y_ref,
                                                                  int n) {
  __shared__ double s_tab[kExpTab];
  fill_exp_tab(s_tab);
  __syncthreads();
  for (int i = blockIdx.x * kSmpThreads + threadIdx.x; i < n; i += gridDim.x * kSmpThreads) {
    const double v = x[i];
    y_tbl[i] = exp_fixup(v, exp_tbl(v, s_tab), s_tab);
    y_ref[i] = exp(v);
  }
}

}  // namespace

cudaError_t launch_exp64_probe(const double* x, double* y_tbl, double* y_ref, int n, cudaStream_t st) {
  const int grid = (n + kSmpThreads - 1) / kSmpThreads < 1184 ? (n + kSmpThreads - 1) / kSmpThreads : 1184;
  exp64_probe_kernel<<<grid, kSmpThreads, 0, st>>>(x, y_tbl, y_ref, n);
  return cudaGetLastError();
}

SamplePlan plan_sampling(int32_t nseq, int32_t gamma, int32_t vocab, int32_t elt) {
  SamplePlan pl{};
  pl.nseq = nseq;
  pl.nrows = nseq * (gamma > 0 ? 2 * gamma + 1 : 1);
  // pass 1 (streamed, no shared memory): at most 40960 elements per CTA, and
  // no more CTAs than fit at once unless the rows need them; at least 256
  // elements per CTA
  const int max_per_cta = kSmpThreads * 160;
  int c1 = (vocab + max_per_cta - 1) / max_per_cta;
  const int want = 148 * kStatsCtasPerSm / pl.nrows;
  if (want > c1) c1 = want;
  const int cap = (vocab + 255) / 256;
  if (c1 > cap) c1 = cap;
  if (c1 < 1) c1 = 1;
  pl.ch1 = (int)align_up((size_t)((vocab + c1 - 1) / c1), 8);
  if (pl.ch1 > max_per_cta) pl.ch1 = max_per_cta;
  pl.c1 = (vocab + pl.ch1 - 1) / pl.ch1;
  // pass 2 (staged): at least 2048 elements per CTA; a chunk is 8 warp
  // segments whose length is a multiple of 32 lanes x 8 elements.
  // Speculative draws (two rows per CTA), and plain draws (one row) whose
  // rows alone fill the GPU: no more CTAs than fit at once (three per SM),
  // unless a chunk would stage more than 72 KB. Fewer plain rows: about 4
  // CTAs per SM, at most 8192 elements each (smaller chunks overlap one CTA's
  // copy with another's arithmetic, which measured faster there).
  const int cap2 = (vocab + 2047) / 2048;
  int c2;
  if (gamma > 0 || nseq >= 148 * kDrawCtasPerSm) {
    const int max_chunk = 72 * 1024 / ((gamma > 0 ? 2 : 1) * elt) / 2048 * 2048;
    c2 = 148 * kDrawCtasPerSm / nseq;
    if (c2 > cap2) c2 = cap2;
    if (c2 < (vocab + max_chunk - 1) / max_chunk) c2 = (vocab + max_chunk - 1) / max_chunk;
  } else {
    c2 = (148 * 4 + nseq - 1) / nseq;
    if (c2 > cap2) c2 = cap2;
    if (c2 < (vocab + 8191) / 8192) c2 = (vocab + 8191) / 8192;
  }
  if (c2 < 1) c2 = 1;
  pl.ch2 = (int)align_up((size_t)((vocab + c2 - 1) / c2), (size_t)kWarpSegs * 32 * 8);
  pl.c2 = (vocab + pl.ch2 - 1) / pl.ch2;
  size_t off = kWsHeader;
  pl.off_tk_row = off;
  off = align_up(off + sizeof(uint32_t) * pl.nrows, 16);
  pl.off_tk_seq1 = off;
  off = align_up(off + sizeof(uint32_t) * nseq, 16);
  pl.off_tk_seq2 = off;
  off = align_up(off + sizeof(uint32_t) * nseq, 16);
  pl.off_tk_seq3 = off;
  off = align_up(off + sizeof(uint32_t) * nseq, 16);
  pl.memset_bytes = off;
  pl.off_j = off;
  off = align_up(off + sizeof(int32_t) * nseq, 256);
  pl.off_part1 = off;
  off = align_up(off + sizeof(Part1) * (size_t)pl.nrows * pl.c1, 256);
  pl.off_stats = off;
  off = align_up(off + sizeof(double) * 2 * (size_t)pl.nrows, 256);
  pl.off_znorm = off;
  off = align_up(off + sizeof(double) * 2 * (size_t)nseq, 256);
  pl.off_zpart = off;
  off = align_up(off + sizeof(double) * 2 * (size_t)nseq * pl.c2, 256);
  pl.off_wpart = off;
  off = align_up(off + sizeof(double) * kWarpSegs * (size_t)nseq * pl.c2, 256);
  pl.off_cmax = off;
  off = align_up(off + sizeof(float) * (size_t)nseq * pl.c2, 256);
  pl.ws_bytes = off;
  return pl;
}

void bind_sample_workspace(SampleParams* p, const SamplePlan& pl, void* ws) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  p->status = reinterpret_cast<uint32_t*>(w);
  p->tk_row = reinterpret_cast<uint32_t*>(w + pl.off_tk_row);
  p->tk_seq1 = reinterpret_cast<uint32_t*>(w + pl.off_tk_seq1);
  p->tk_seq2 = reinterpret_cast<uint32_t*>(w + pl.off_tk_seq2);
  p->tk_seq3 = reinterpret_cast<uint32_t*>(w + pl.off_tk_seq3);
  p->jsel = reinterpret_cast<int32_t*>(w + pl.off_j);
  p->part1 = w + pl.off_part1;
  p->stats = reinterpret_cast<double*>(w + pl.off_stats);
  p->znorm = reinterpret_cast<double*>(w + pl.off_znorm);
  p->zpart = reinterpret_cast<double*>(w + pl.off_zpart);
  p->wpart = reinterpret_cast<double*>(w + pl.off_wpart);
  p->cmax = reinterpret_cast<float*>(w + pl.off_cmax);
  p->c1 = pl.c1;
  p->ch1 = pl.ch1;
  p->c2 = pl.c2;
  p->ch2 = pl.ch2;
}

cudaError_t launch_sampling(const SampleParams& p, s3r_dtype dt, bool spec, cudaStream_t st) {
  if (dt == S3R_BF16) return spec ? launch_typed<__nv_bfloat16, true>(p, st) : launch_typed<__nv_bfloat16, false>(p, st);
  return spec ? launch_typed<float, true>(p, st) : launch_typed<float, false>(p, st);
}

}  // namespace s3r
