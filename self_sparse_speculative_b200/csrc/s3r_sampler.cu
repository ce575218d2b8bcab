// Exact speculative sampling of one S3R round, vocab-wide, on the GPU.
//
// S3R page (weekinpapers.com, Abstract): tokens are committed by "exact
// speculative sampling" so that responses follow the dense policy. The rule
// (speculative-sampling papers on the mlsanity.com reference list; restated
// on the ai.info SpecRoll page): accept draft x_i iff u < p_i(x_i)/q_i(x_i);
// at the first rejection j draw from norm(max(p_j - q_j, 0)); if all gamma
// drafts pass, draw a bonus token from p_gamma.
//
// Pass 1 (grid: vocab chunks x rows): every CTA holds its chunk of one logits
// row in registers (one HBM read), reduces its max, then sums exp((x - max)/T)
// with float32 exponentials into float64. The last CTA of a row (atomic
// ticket) merges the chunk partials into the row's (max, Z); the last row of
// a sequence takes the gamma accept/reject tests (one lane each) in float64.
// Pass 2a (residual sequences only): the exact float64 normalisers of the
// two rows the residual is drawn from (float64 exponentials).
// Pass 2b (grid: vocab chunks x sequences): float64 draw weights, summed per
// warp segment; the last CTA of a sequence finds the chunk, then the warp
// segment holding u * total, and one warp scans it for the drawn token. Every
// draw is decided in float64 on both sides, so it is exact up to the order of
// the float64 sums.
// The drafter's own draw (s3r_sample_tokens) is pass 1 + pass 2b in "plain"
// mode: one row per draw, weights exp((x - max)/T).
#include <cuda_bf16.h>

#include <cmath>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kSmpThreads = 256;
constexpr int kSmpWarps = kSmpThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWarpSegs = kSmpWarps;         // pass-2 chunk = 8 contiguous warp segments

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
      const double* sd = p.stats + 2 * ((size_t)b * per + R + lane);
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
template <typename T, bool SPEC, bool VEC>
__global__ void __launch_bounds__(kSmpThreads) rowstats_kernel(const SampleParams p) {
  __shared__ float s_redf[kSmpWarps];
  __shared__ double s_redd[kSmpWarps];
  __shared__ int s_last;
  using IO = LogitIO<T>;
  constexpr int E = IO::kPerVec * IO::kVecs;     // elements per thread
  const int row = blockIdx.y, c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* src = row_ptr<T>(p, SPEC, row);
  const int beg = c * p.ch1;
  const int end = min(p.vocab, beg + p.ch1);
  float x[E];
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
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int k = 0; k < E; ++k) mx[k & 3] = fmaxf(mx[k & 3], x[k]);
  const float M = block_max(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), s_redf);
  const float k2 = kLog2e * p.inv_temp;
  double s4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int k = 0; k < E; ++k) s4[k & 3] += static_cast<double>(ex2((x[k] - M) * k2));
  double s = warp_sum_d((s4[0] + s4[1]) + (s4[2] + s4[3]));
  if (lane == 0) s_redd[warp] = s;
  __syncthreads();
  if (tid == 0) {
    double S = 0.0;
    for (int w = 0; w < kSmpWarps; ++w) S += s_redd[w];
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
  if constexpr (SPEC) {
    const int per = 2 * p.gamma + 1;
    const int b = row / per;
    int last = 0;
    if (lane == 0) {
      __threadfence();
      last = atomicAdd(p.tk_seq1 + b, 1u) == (unsigned)(per - 1);
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence();
      if (lane == 0) p.tk_seq1[b] = 0u;
      decide<T>(p, b);
    }
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
__device__ DrawRows draw_rows(const SampleParams& p, int s, int j, bool exact_z) {
  DrawRows w;
  w.iZp = 1.0;
  w.iZq = 1.0;
  w.qrow = nullptr;
  w.Mq = 0.0;
  if (!SPEC) {
    w.prow = static_cast<const T*>(p.target) + (size_t)s * p.vocab;
    w.Mp = p.stats[2 * (size_t)s];
    return w;
  }
  const int per = 2 * p.gamma + 1, R = p.gamma + 1;
  w.prow = static_cast<const T*>(p.target) + ((size_t)s * R + j) * p.vocab;
  w.Mp = p.stats[2 * ((size_t)s * per + j)];
  if (j < p.gamma) {
    w.qrow = static_cast<const T*>(p.draft) + ((size_t)s * p.gamma + j) * p.vocab;
    w.Mq = p.stats[2 * ((size_t)s * per + R + j)];
    if (exact_z) {
      w.iZp = 1.0 / __ldcg(p.znorm + 2 * (size_t)s);
      w.iZq = 1.0 / __ldcg(p.znorm + 2 * (size_t)s + 1);
    }
  }
  return w;
}

// float64 draw weights of n consecutive elements starting at e
template <typename T, bool VEC>
__device__ __forceinline__ void load_vals(const T* row, int e, int n, float* v) {
  using IO = LogitIO<T>;
  if constexpr (VEC) {
    IO::unpack(ldg_stream16(row + e), v);
  } else {
    for (int t = 0; t < IO::kPerVec; ++t) v[t] = t < n ? IO::at(row, e + t) : 0.f;
  }
}

template <typename T, bool VEC>
__device__ __forceinline__ void weights(const DrawRows& w, int e, int n, double invT, double* out) {
  using IO = LogitIO<T>;
  float a[IO::kPerVec], b[IO::kPerVec];
  load_vals<T, VEC>(static_cast<const T*>(w.prow), e, n, a);
  if (w.qrow) load_vals<T, VEC>(static_cast<const T*>(w.qrow), e, n, b);
#pragma unroll
  for (int t = 0; t < IO::kPerVec; ++t) {
    double wt = 0.0;
    if (t < n) {
      const double pe = exp((static_cast<double>(a[t]) - w.Mp) * invT) * w.iZp;
      if (w.qrow) {
        const double qe = exp((static_cast<double>(b[t]) - w.Mq) * invT) * w.iZq;
        wt = pe > qe ? pe - qe : 0.0;
      } else {
        wt = pe;
      }
    }
    out[t] = wt;
  }
}

// Pass 2a: exact float64 normalisers of the residual's two rows.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kSmpThreads) znorm_kernel(const SampleParams p) {
  __shared__ double s_red[2][kSmpWarps];
  __shared__ int s_last;
  using IO = LogitIO<T>;
  const int s = blockIdx.y, c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = p.jsel[s];
  if (j >= p.gamma) return;                              // bonus draw: no residual (uniform per sequence)
  DrawRows w = draw_rows<T, true>(p, s, j, false);
  const int beg = c * p.ch2, end = min(p.vocab, beg + p.ch2);
  double zt = 0.0, zd = 0.0;
  for (int e = beg + tid * IO::kPerVec; e < end; e += kSmpThreads * IO::kPerVec) {
    const int n = min(IO::kPerVec, end - e);
    float a[IO::kPerVec], b[IO::kPerVec];
    load_vals<T, VEC>(static_cast<const T*>(w.prow), e, n, a);
    load_vals<T, VEC>(static_cast<const T*>(w.qrow), e, n, b);
#pragma unroll
    for (int t = 0; t < IO::kPerVec; ++t) {
      if (t < n) {
        zt += exp((static_cast<double>(a[t]) - w.Mp) * p.inv_temp_d);
        zd += exp((static_cast<double>(b[t]) - w.Mq) * p.inv_temp_d);
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
    p.znorm[2 * (size_t)s + 1] = b;
    p.tk_seq3[s] = 0u;
  }
}

// One warp scans [beg, end) from running sum `base` for the first k whose
// running sum exceeds thr. Returns k, or -1 - (last index with weight > 0).
template <typename T, bool VEC>
__device__ int warp_scan_find(const DrawRows& w, int beg, int end, double base, double thr, double invT) {
  using IO = LogitIO<T>;
  constexpr int PV = IO::kPerVec;
  const int lane = threadIdx.x & 31;
  int last_pos = -1;
  double run = base;
  for (int e0 = beg; e0 < end; e0 += 32 * PV) {
    const int e = e0 + lane * PV;
    double wv[PV];
    const int n = max(0, min(PV, end - e));
    if (n > 0) weights<T, VEC>(w, e, n, invT, wv);
    else
#pragma unroll
      for (int t = 0; t < PV; ++t) wv[t] = 0.0;
    double loc = 0.0;
#pragma unroll
    for (int t = 0; t < PV; ++t) loc += wv[t];
    double incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const double before = run + incl - loc;
    int hit = -1, lp = -1;
    double r = before;
#pragma unroll
    for (int t = 0; t < PV; ++t) {
      r += wv[t];
      if (wv[t] > 0.0) lp = e + t;
      if (hit < 0 && r > thr) hit = e + t;
    }
    const unsigned m = __ballot_sync(0xffffffffu, hit >= 0);
    if (m) return __shfl_sync(0xffffffffu, hit, __ffs(m) - 1);
    const unsigned mp = __ballot_sync(0xffffffffu, lp >= 0);
    if (mp) last_pos = __shfl_sync(0xffffffffu, lp, 31 - __clz(mp));
    run = __shfl_sync(0xffffffffu, run + incl, 31);
  }
  return -1 - last_pos;
}

// Pass 2b: the draw.
template <typename T, bool SPEC, bool VEC>
__global__ void __launch_bounds__(kSmpThreads) draw_kernel(const SampleParams p) {
  __shared__ double s_w[kSmpWarps];
  __shared__ int s_last;
  using IO = LogitIO<T>;
  constexpr int PV = IO::kPerVec;
  const int s = blockIdx.y, c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = SPEC ? p.jsel[s] : 0;
  const DrawRows w = draw_rows<T, SPEC>(p, s, j, true);
  const int cbeg = c * p.ch2, cend = min(p.vocab, cbeg + p.ch2);
  const int seg = p.ch2 / kWarpSegs;                     // elements per warp segment
  const int sbeg = min(cend, cbeg + warp * seg), send = min(cend, sbeg + seg);
  double acc = 0.0;
  for (int e = sbeg + lane * PV; e < send; e += 32 * PV) {
    double wv[PV];
    weights<T, VEC>(w, e, min(PV, send - e), p.inv_temp_d, wv);
#pragma unroll
    for (int t = 0; t < PV; ++t) acc += wv[t];
  }
  acc = warp_sum_d(acc);
  if (lane == 0) {
    p.wpart[((size_t)s * p.c2 + c) * kWarpSegs + warp] = acc;
    s_w[warp] = acc;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(p.tk_seq2 + s, 1u) == (unsigned)(p.c2 - 1);
  }
  __syncthreads();
  if (!s_last || warp != 0) return;
  __threadfence();
  const int R = p.gamma + 1;
  const double u = SPEC ? static_cast<double>(p.u_sample[(size_t)s * R + j]) : static_cast<double>(p.u_sample[s]);
  const double* wp = p.wpart + (size_t)s * p.c2 * kWarpSegs;
  const int nseg = p.c2 * kWarpSegs;
  // total of all segments, then the first segment whose running sum passes thr
  double tot = 0.0;
  for (int i = lane; i < nseg; i += 32) tot += __ldcg(wp + i);
  tot = warp_sum_d(tot);
  int k = -1;
  if (tot > 0.0) {
    const double thr = u * tot;
    double run = 0.0;
    int sel = -1, lastpos = -1;
    double sel_base = 0.0;
    for (int i0 = 0; i0 < nseg && sel < 0; i0 += 32) {
      const int i = i0 + lane;
      const double v = i < nseg ? __ldcg(wp + i) : 0.0;
      double incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned m = __ballot_sync(0xffffffffu, run + incl > thr && v > 0.0);
      if (m) {
        const int src = __ffs(m) - 1;
        sel = i0 + src;
        sel_base = __shfl_sync(0xffffffffu, run + incl - v, src);
      }
      const unsigned mp = __ballot_sync(0xffffffffu, v > 0.0);
      if (mp) lastpos = i0 + 31 - __clz(mp);
      run = __shfl_sync(0xffffffffu, run + incl, 31);
    }
    if (sel < 0) {                                       // rounding left no crossing: last segment with weight
      sel = lastpos;
      sel_base = 0.0;
      for (int i = lane; i < sel; i += 32) sel_base += __ldcg(wp + i);
      sel_base = warp_sum_d(sel_base);
    }
    if (sel >= 0) {
      const int cc = sel / kWarpSegs, ww = sel - cc * kWarpSegs;
      const int b0 = min(p.vocab, cc * p.ch2 + ww * seg), b1 = min(min(p.vocab, cc * p.ch2 + p.ch2), b0 + seg);
      k = warp_scan_find<T, VEC>(w, b0, b1, sel_base, thr, p.inv_temp_d);
      if (k < 0) k = -1 - k;                            // last positive weight of the segment
    }
  } else if (SPEC && w.qrow) {
    // all-zero residual (p_j == q_j after rounding): draw from p_j instead
    DrawRows wb = w;
    wb.qrow = nullptr;
    wb.iZp = 1.0;
    double total = 0.0;
    for (int e = lane * PV; e < p.vocab; e += 32 * PV) {
      double wv[PV];
      weights<T, VEC>(wb, e, min(PV, p.vocab - e), p.inv_temp_d, wv);
#pragma unroll
      for (int t = 0; t < PV; ++t) total += wv[t];
    }
    total = warp_sum_d(total);
    k = warp_scan_find<T, VEC>(wb, 0, p.vocab, 0.0, u * total, p.inv_temp_d);
    if (k < 0) k = -1 - k;
  }
  if (lane == 0) {
    if (k < 0) k = 0;
    if (SPEC) p.out_tokens[(size_t)s * R + j] = k;
    else p.out_tokens[s] = k;
    p.tk_seq2[s] = 0u;
  }
}

template <typename T, bool SPEC>
cudaError_t launch_typed(const SampleParams& p, cudaStream_t st) {
  const int per = SPEC ? 2 * p.gamma + 1 : 1;
  const int nrows = p.nseq * per;
  const bool vec = (((size_t)p.vocab * sizeof(T)) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(p.target) % 16 == 0) &&
                   (!SPEC || reinterpret_cast<uintptr_t>(p.draft) % 16 == 0);
  dim3 g1(p.c1, nrows), g2(p.c2, p.nseq);
  if (vec) rowstats_kernel<T, SPEC, true><<<g1, kSmpThreads, 0, st>>>(p);
  else rowstats_kernel<T, SPEC, false><<<g1, kSmpThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (SPEC) {
    if (vec) znorm_kernel<T, true><<<g2, kSmpThreads, 0, st>>>(p);
    else znorm_kernel<T, false><<<g2, kSmpThreads, 0, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (vec) draw_kernel<T, SPEC, true><<<g2, kSmpThreads, 0, st>>>(p);
  else draw_kernel<T, SPEC, false><<<g2, kSmpThreads, 0, st>>>(p);
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
  // pass 2: about 4 CTAs per SM, at least 2048 elements per CTA; a chunk is
  // 8 warp segments whose length is a multiple of 32 lanes x 8 elements
  int c2 = (target + nseq - 1) / nseq;
  const int cap2 = (vocab + 2047) / 2048;
  if (c2 > cap2) c2 = cap2;
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
