// Exact speculative sampling of one S3R round, vocab-wide, on the GPU.
//
// S3R page (weekinpapers.com, Abstract): tokens are committed by "exact
// speculative sampling" so that responses follow the dense policy. The rule
// (speculative-sampling papers on the mlsanity.com reference list; restated
// on the ai.info SpecRoll page): accept draft x_i iff u < p_i(x_i)/q_i(x_i);
// at the first rejection j draw from norm(max(p_j - q_j, 0)); if all gamma
// drafts pass, draw a bonus token from p_gamma.
//
// Pass 1 (grid: vocab chunks x rows): every CTA holds its chunk of one
// logits row in registers (one HBM read), reduces its max, then sums
// exp((x - max)/T) in float64. The last CTA of a row (atomic ticket) merges
// the chunk partials into the row's (max, Z) in float64; the last row of a
// sequence to finish takes the accept/reject decisions in float64.
// Pass 2 (grid: vocab chunks x sequences): every CTA sums its chunk of the
// residual (or bonus) weights in float64; the last CTA of a sequence locates
// the chunk holding u * total and scans it for the drawn token.
// The drafter's own draw (s3r_sample_tokens) is the same two passes in
// "plain" mode: one row per draw, weights softmax(logits / T).
#include <cuda_bf16.h>

#include <cmath>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kSmpThreads = 256;
constexpr int kSmpWarps = kSmpThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

struct Part1 {
  float m;
  float pad;
  double s;
};

template <typename T> struct LogitIO;
template <> struct LogitIO<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  static constexpr int kVecs = 8;           // 16-byte vectors per thread in pass 1
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
  static constexpr int kVecs = 16;
  __device__ static float at(const float* p, size_t i) { return p[i]; }
  __device__ static void unpack(const uint4& v, float* x) {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
  }
};

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ float block_max(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float r = s_red[0];
  for (int w = 1; w < kSmpWarps; ++w) r = fmaxf(r, s_red[w]);
  __syncthreads();
  return r;
}
__device__ double block_sum(double v, double* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  double r = 0.0;
  for (int w = 0; w < kSmpWarps; ++w) r += s_red[w];
  __syncthreads();
  return r;
}
// Exclusive prefix sum of doubles over the CTA; *total gets the sum.
__device__ double block_exclusive_scan_d(double v, double* total, double* s_red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_red[warp] = x;
  __syncthreads();
  double before = 0.0, tot = 0.0;
  for (int w = 0; w < kSmpWarps; ++w) {
    if (w < warp) before += s_red[w];
    tot += s_red[w];
  }
  __syncthreads();
  *total = tot;
  return before + x - v;
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

// accept/reject decisions of sequence b (one thread)
template <typename T>
__device__ void decide(const SampleParams& p, int b) {
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  int j = p.gamma;
  for (int i = 0; i < p.gamma; ++i) {
    const int x = p.draft_tokens[(size_t)b * p.gamma + i];
    double ratio = 0.0;
    if (x >= 0 && x < p.vocab) {
      // statistics written by other CTAs of this grid: read through L2
      const double* st = p.stats + 2 * ((size_t)b * per + i);
      const double* sd = p.stats + 2 * ((size_t)b * per + R + i);
      const double lt = LogitIO<T>::at(static_cast<const T*>(p.target) + ((size_t)b * R + i) * p.vocab, x);
      const double ld = LogitIO<T>::at(static_cast<const T*>(p.draft) + ((size_t)b * p.gamma + i) * p.vocab, x);
      const double px = exp((lt - __ldcg(st)) * p.inv_temp_d) / __ldcg(st + 1);
      const double qx = exp((ld - __ldcg(sd)) * p.inv_temp_d) / __ldcg(sd + 1);
      ratio = qx > 0.0 ? px / qx : 0.0;
    } else {
      flag_status(p.status, S3R_DEV_BAD_TOKEN_ID);
    }
    if (!(static_cast<double>(p.u_accept[(size_t)b * p.gamma + i]) < ratio)) { j = i; break; }
  }
  for (int i = 0; i < R; ++i) {
    if (i < j) p.out_tokens[(size_t)b * R + i] = p.draft_tokens[(size_t)b * p.gamma + i];
    else if (i > j) p.out_tokens[(size_t)b * R + i] = -1;
  }
  p.num_accepted[b] = j;
  p.jsel[b] = j;
}

// ---------------------------------------------------------------- pass 1
template <typename T, bool SPEC, bool VEC>
__global__ void __launch_bounds__(kSmpThreads) rowstats_kernel(const SampleParams p) {
  __shared__ float s_redf[kSmpWarps];
  __shared__ double s_redd[kSmpWarps];
  __shared__ int s_last;
  using IO = LogitIO<T>;
  constexpr int E = IO::kPerVec * IO::kVecs;     // elements per thread
  const int row = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  const T* src = row_ptr<T>(p, SPEC, row);
  const int beg = c * p.ch1;
  const int end = min(p.vocab, beg + p.ch1);
  float x[E];
  float mx = -INFINITY;
  if constexpr (VEC) {
#pragma unroll
    for (int k = 0; k < IO::kVecs; ++k) {
      const int e0 = beg + (tid + k * kSmpThreads) * IO::kPerVec;
      if (e0 < end) {
        IO::unpack(ldg_stream16(src + e0), x + k * IO::kPerVec);
      } else {
#pragma unroll
        for (int t = 0; t < IO::kPerVec; ++t) x[k * IO::kPerVec + t] = -INFINITY;
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int e = beg + tid + k * kSmpThreads;
      x[k] = e < end ? IO::at(src, e) : -INFINITY;
    }
  }
#pragma unroll
  for (int k = 0; k < E; ++k) mx = fmaxf(mx, x[k]);
  const float M = block_max(mx, s_redf);
  const float k2 = kLog2e * p.inv_temp;
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < E; ++k) s += static_cast<double>(ex2((x[k] - M) * k2));
  const double S = block_sum(s, s_redd);
  if (tid == 0) {
    Part1* part = static_cast<Part1*>(p.part1) + (size_t)row * p.c1 + c;
    part->m = M;
    part->s = S;
    __threadfence();
    s_last = (atomicAdd(p.tk_row + row, 1u) == (unsigned)(p.c1 - 1));
  }
  __syncthreads();
  if (!s_last) return;
  // last CTA of the row: merge chunk partials in float64
  if (tid == 0) {
    __threadfence();
    const Part1* part = static_cast<const Part1*>(p.part1) + (size_t)row * p.c1;
    float Mr = -INFINITY;
    for (int i = 0; i < p.c1; ++i) Mr = fmaxf(Mr, __ldcg(&part[i].m));
    double Z = 0.0;
    for (int i = 0; i < p.c1; ++i) {
      const float mi = __ldcg(&part[i].m);
      if (mi == -INFINITY) continue;
      Z += __ldcg(&part[i].s) * exp((static_cast<double>(mi) - static_cast<double>(Mr)) * p.inv_temp_d);
    }
    p.stats[2 * (size_t)row] = Mr;
    p.stats[2 * (size_t)row + 1] = Z;
    p.tk_row[row] = 0u;
    if constexpr (SPEC) {
      const int per = 2 * p.gamma + 1;
      const int b = row / per;
      __threadfence();
      if (atomicAdd(p.tk_seq1 + b, 1u) == (unsigned)(per - 1)) {
        __threadfence();
        p.tk_seq1[b] = 0u;
        decide<T>(p, b);
      }
    }
  }
}

// ---------------------------------------------------------------- pass 2
struct DrawRows {
  const void* prow;   // weights' p row
  const void* qrow;   // residual: q row, else null
  double Mp, Zp, Mq, Zq;
};

template <typename T>
__device__ __forceinline__ double weight(const DrawRows& w, int e, double invT) {
  const double pe = exp((static_cast<double>(LogitIO<T>::at(static_cast<const T*>(w.prow), e)) - w.Mp) * invT) / w.Zp;
  if (!w.qrow) return pe;
  const double qe = exp((static_cast<double>(LogitIO<T>::at(static_cast<const T*>(w.qrow), e)) - w.Mq) * invT) / w.Zq;
  return pe > qe ? pe - qe : 0.0;
}

template <typename T, bool SPEC>
__device__ DrawRows draw_rows(const SampleParams& p, int s, int j) {
  DrawRows w;
  if (!SPEC) {
    w.prow = static_cast<const T*>(p.target) + (size_t)s * p.vocab;
    w.qrow = nullptr;
    w.Mp = p.stats[2 * (size_t)s];
    w.Zp = p.stats[2 * (size_t)s + 1];
    w.Mq = 0.0; w.Zq = 1.0;
    return w;
  }
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  w.prow = static_cast<const T*>(p.target) + ((size_t)s * R + j) * p.vocab;
  w.Mp = p.stats[2 * ((size_t)s * per + j)];
  w.Zp = p.stats[2 * ((size_t)s * per + j) + 1];
  if (j < p.gamma) {
    w.qrow = static_cast<const T*>(p.draft) + ((size_t)s * p.gamma + j) * p.vocab;
    w.Mq = p.stats[2 * ((size_t)s * per + R + j)];
    w.Zq = p.stats[2 * ((size_t)s * per + R + j) + 1];
  } else {
    w.qrow = nullptr;
    w.Mq = 0.0; w.Zq = 1.0;
  }
  return w;
}

// Sum of weights over [beg, end) by the whole CTA.
template <typename T>
__device__ double chunk_sum(const DrawRows& w, int beg, int end, double invT, double* s_red) {
  double acc = 0.0;
  for (int e = beg + threadIdx.x; e < end; e += kSmpThreads) acc += weight<T>(w, e, invT);
  return block_sum(acc, s_red);
}

// Smallest k in [beg, end) with base + sum_{e in [beg, k]} w(e) > thr, by
// contiguous per-thread segments and a block scan; -1 if none.
template <typename T>
__device__ int chunk_search(const DrawRows& w, int beg, int end, double base, double thr, double invT,
                            double* s_red, int* s_int) {
  const int n = end - beg;
  const int per = (n + kSmpThreads - 1) / kSmpThreads;
  const int sb = beg + min(n, (int)threadIdx.x * per), se = min(end, sb + per);
  double loc = 0.0;
  for (int e = sb; e < se; ++e) loc += weight<T>(w, e, invT);
  double tot;
  const double before = block_exclusive_scan_d(loc, &tot, s_red);
  if (threadIdx.x == 0) { s_int[0] = 0x7FFFFFFF; s_int[1] = -1; }
  __syncthreads();
  double run = base + before;
  int found = -1, last_pos = -1;
  for (int e = sb; e < se; ++e) {
    const double we = weight<T>(w, e, invT);
    run += we;
    if (we > 0.0) last_pos = e;
    if (found < 0 && run > thr) found = e;
  }
  if (found >= 0) atomicMin(&s_int[0], found);
  if (last_pos >= 0) atomicMax(&s_int[1], last_pos);
  __syncthreads();
  const int k = s_int[0] != 0x7FFFFFFF ? s_int[0] : -1;
  const int lp = s_int[1];
  __syncthreads();
  return k >= 0 ? k : (lp >= 0 ? -2 - lp : -1);   // -2-lp encodes "none, last positive lp"
}

template <typename T, bool SPEC>
__global__ void __launch_bounds__(kSmpThreads) draw_kernel(const SampleParams p) {
  __shared__ double s_redd[kSmpWarps];
  __shared__ int s_int[2];
  __shared__ int s_last;
  __shared__ int s_chunk;
  __shared__ double s_base, s_thr;
  const int s = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  const int j = SPEC ? p.jsel[s] : 0;
  DrawRows w = draw_rows<T, SPEC>(p, s, j);
  const int beg = c * p.ch2, end = min(p.vocab, beg + p.ch2);
  const double S = chunk_sum<T>(w, beg, end, p.inv_temp_d, s_redd);
  if (tid == 0) {
    p.part2[(size_t)s * p.c2 + c] = S;
    __threadfence();
    s_last = (atomicAdd(p.tk_seq2 + s, 1u) == (unsigned)(p.c2 - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int R = p.gamma + 1;
  const double u = SPEC ? static_cast<double>(p.u_sample[(size_t)s * R + j]) : static_cast<double>(p.u_sample[s]);
  // totals of the chunk sums; an all-zero residual falls back to p_j
  if (tid == 0) {
    double tot = 0.0;
    for (int i = 0; i < p.c2; ++i) tot += __ldcg(p.part2 + (size_t)s * p.c2 + i);
    s_base = tot;
  }
  __syncthreads();
  if (SPEC && s_base <= 0.0 && w.qrow) {
    w.qrow = nullptr;                                     // empty residual: draw from p_j
    for (int i = 0; i < p.c2; ++i) {
      const int b2 = i * p.ch2, e2 = min(p.vocab, b2 + p.ch2);
      const double cs = chunk_sum<T>(w, b2, e2, p.inv_temp_d, s_redd);
      if (tid == 0) p.part2[(size_t)s * p.c2 + i] = cs;
    }
    __syncthreads();
  }
  if (tid == 0) {
    double tot = 0.0;
    for (int i = 0; i < p.c2; ++i) tot += __ldcg(p.part2 + (size_t)s * p.c2 + i);
    const double thr = u * tot;
    double run = 0.0;
    int cstar = -1, lastpos = -1;
    double base = 0.0;
    for (int i = 0; i < p.c2; ++i) {
      const double ci = __ldcg(p.part2 + (size_t)s * p.c2 + i);
      if (ci > 0.0) { lastpos = i; }
      if (cstar < 0 && run + ci > thr) { cstar = i; base = run; }
      run += ci;
    }
    if (cstar < 0) {            // rounding left no crossing: last chunk with weight
      cstar = lastpos < 0 ? 0 : lastpos;
      base = 0.0;
      for (int i = 0; i < cstar; ++i) base += __ldcg(p.part2 + (size_t)s * p.c2 + i);
    }
    s_chunk = cstar;
    s_base = base;
    s_thr = thr;
    p.tk_seq2[s] = 0u;
  }
  __syncthreads();
  const int cb = s_chunk * p.ch2, ce = min(p.vocab, cb + p.ch2);
  int k = chunk_search<T>(w, cb, ce, s_base, s_thr, p.inv_temp_d, s_redd, s_int);
  if (tid == 0) {
    if (k <= -2) k = -2 - k;          // no crossing inside: last positive weight
    if (k < 0) k = cb;                // no weight at all (cannot happen for a distribution)
    if (SPEC) p.out_tokens[(size_t)s * R + j] = k;
    else p.out_tokens[s] = k;
  }
}

template <typename T, bool SPEC>
cudaError_t launch_typed(const SampleParams& p, cudaStream_t st) {
  const int per = SPEC ? 2 * p.gamma + 1 : 1;
  const int nrows = p.nseq * per;
  const bool vec = (((size_t)p.vocab * sizeof(T)) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(p.target) % 16 == 0) &&
                   (!SPEC || reinterpret_cast<uintptr_t>(p.draft) % 16 == 0);
  dim3 g1(p.c1, nrows);
  if (vec) rowstats_kernel<T, SPEC, true><<<g1, kSmpThreads, 0, st>>>(p);
  else rowstats_kernel<T, SPEC, false><<<g1, kSmpThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(p.c2, p.nseq);
  draw_kernel<T, SPEC><<<g2, kSmpThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

SamplePlan plan_sampling(int32_t nseq, int32_t gamma, int32_t vocab) {
  SamplePlan pl{};
  pl.nseq = nseq;
  pl.nrows = nseq * (gamma > 0 ? 2 * gamma + 1 : 1);
  // pass 1: at most 64 register-resident elements per thread (16384 per CTA),
  // about 4 CTAs per SM overall, at least 256 elements per CTA
  const int max_per_cta = kSmpThreads * 64;
  const int target = 148 * 4;
  int c1 = (vocab + max_per_cta - 1) / max_per_cta;
  const int want = (target + pl.nrows - 1) / pl.nrows;
  if (want > c1) c1 = want;
  const int cap = (vocab + 255) / 256;
  if (c1 > cap) c1 = cap;
  if (c1 < 1) c1 = 1;
  pl.ch1 = (int)align_up((size_t)((vocab + c1 - 1) / c1), 8);
  if (pl.ch1 > max_per_cta) pl.ch1 = max_per_cta;
  pl.c1 = (vocab + pl.ch1 - 1) / pl.ch1;
  // pass 2: about 4 CTAs per SM, at least 1024 elements per CTA
  int c2 = (target + nseq - 1) / nseq;
  const int cap2 = (vocab + 1023) / 1024;
  if (c2 > cap2) c2 = cap2;
  if (c2 < 1) c2 = 1;
  pl.ch2 = (int)align_up((size_t)((vocab + c2 - 1) / c2), 8);
  pl.c2 = (vocab + pl.ch2 - 1) / pl.ch2;
  size_t off = kWsHeader;
  pl.off_tk_row = off;
  off = align_up(off + sizeof(uint32_t) * pl.nrows, 16);
  pl.off_tk_seq1 = off;
  off = align_up(off + sizeof(uint32_t) * nseq, 16);
  pl.off_tk_seq2 = off;
  off = align_up(off + sizeof(uint32_t) * nseq, 16);
  pl.memset_bytes = off;
  pl.off_j = off;
  off = align_up(off + sizeof(int32_t) * nseq, 256);
  pl.off_part1 = off;
  off = align_up(off + sizeof(Part1) * (size_t)pl.nrows * pl.c1, 256);
  pl.off_stats = off;
  off = align_up(off + sizeof(double) * 2 * (size_t)pl.nrows, 256);
  pl.off_part2 = off;
  off = align_up(off + sizeof(double) * (size_t)nseq * pl.c2, 256);
  pl.ws_bytes = off;
  return pl;
}

cudaError_t launch_sampling(const SampleParams& p, s3r_dtype dt, bool spec, cudaStream_t st) {
  if (dt == S3R_BF16) return spec ? launch_typed<__nv_bfloat16, true>(p, st) : launch_typed<__nv_bfloat16, false>(p, st);
  return spec ? launch_typed<float, true>(p, st) : launch_typed<float, false>(p, st);
}

}  // namespace s3r
