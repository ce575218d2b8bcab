// Tree verification of a round: exact speculative sampling walked over a
// token tree (the ai.info SpecRoll page: sparse-tree verification whose
// node budget follows the number of unfinished responses; exact rejection
// sampling with the target-residual fallback at every visited node, so the
// committed tokens keep the target distribution).
//
// Rule, per sequence (nodes 0..R-1, parent[0] = -1, parents precede their
// children): p_v = softmax(target[v] / T) and q_v = softmax(draft[v] / T),
// the distribution node v's children were drawn from. At node v the
// children c are tested in ascending order: accept c iff
// u_accept[c] < p'(x_c) / q_v(x_c), with p' = p_v at first and, after each
// rejection, p' <- max(p' - q_v, 0) normalised (p' renormalised where that
// residual is zero everywhere). An accepted child commits its token and
// becomes v; when no child is accepted, or v has none, the token drawn from
// p' with u_sample[v] (inverse CDF: the smallest k whose running sum exceeds
// u times the total) is committed and the walk ends.
//
// One thread-block cluster of ncl <= 8 CTAs per sequence (the largest size
// whose clusters all fit on the GPU at once); CTA r owns the vocab slice r. The walk is sequential, each of its vocab-wide quantities a
// pass over the slices whose per-CTA results every CTA stores into every
// other CTA's shared memory (st.shared::cluster) before a cluster barrier;
// every CTA then combines them in rank order, so all of them hold identical
// values and take identical decisions without another round trip. When the
// rows are 16-byte aligned, each visited node's two row slices are
// bulk-copied into shared memory once (cp.async.bulk, no multicast) and every
// pass at that node reads them there.
//
// Precision. The accept tests read p'(x_c) and q_v(x_c) at single tokens in
// float64; the row normalisers they divide by (and those of the residual
// chain) are float64 sums of float32 exponentials, as for the chain sampler's
// tests. The final draw needs exact weights: at a leaf they are the
// unnormalised float64 exponentials exp((t - max) / T) (the draw is
// invariant to scale); at a node that rejected children the normalisers and
// the residual chain are first recomputed with float64 exponentials
// (exp_tbl), then the weights.
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

#include "s3r_device.cuh"
#include "s3r_exp64.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kTreeThreads = 512;
constexpr int kTreeWarps = kTreeThreads / 32;
constexpr int kTreeMaxCluster = 8;
constexpr size_t kTreeStageMax = 200 * 1024;      // bytes of a CTA's two staged row slices, at most
constexpr uint32_t kTreePiece = 16384;             // bytes per bulk-copy instruction

struct TreeParams {
  const void* target;       // [S, R, V]
  const void* draft;        // [S, R, V]
  const int32_t* tokens;    // [S, R] token of each node (node 0: unused)
  const int32_t* parents;   // [S, R]
  const float* u_accept;    // [S, R] (node 0: unused)
  const float* u_sample;    // [S, R]
  int32_t* out_tokens;      // [S, R]
  int32_t* num_accepted;    // [S]
  int32_t* path;            // [S, R] or null
  int32_t nseq, nodes, vocab;
  int32_t ncl;              // CTAs per cluster (one cluster per sequence)
  int32_t stage;            // 1: row slices staged in shared memory (rows 16-byte aligned)
  double inv_temp;
  uint32_t* status;
};

// PV logits from element i of a row as one 16-byte word (PV > 1: i a multiple
// of PV, the row 16-byte aligned), and their float values.
template <typename T, int PV> struct TreeLoad;
template <> struct TreeLoad<__nv_bfloat16, 8> {
  static __device__ __forceinline__ uint4 raw(const __nv_bfloat16* row, int i) {
    return __ldg(reinterpret_cast<const uint4*>(row + i));
  }
  static __device__ __forceinline__ void cvt(const uint4& u, float* o) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = __uint_as_float(w[k] << 16);
      o[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};
template <> struct TreeLoad<float, 4> {
  static __device__ __forceinline__ uint4 raw(const float* row, int i) {
    return __ldg(reinterpret_cast<const uint4*>(row + i));
  }
  static __device__ __forceinline__ void cvt(const uint4& u, float* o) {
    o[0] = __uint_as_float(u.x); o[1] = __uint_as_float(u.y); o[2] = __uint_as_float(u.z); o[3] = __uint_as_float(u.w);
  }
};
template <typename T> struct TreeLoad<T, 1> {
  static __device__ __forceinline__ uint4 raw(const T* row, int i) {
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (sizeof(T) == 2) u.x = static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(row) + i)) << 16;
    else u.x = __float_as_uint(__ldg(row + i));
    return u;
  }
  static __device__ __forceinline__ void cvt(const uint4& u, float* o) { o[0] = __uint_as_float(u.x); }
};
// PV logits at p (global or shared memory; 16-byte aligned when PV > 1)
template <typename T, int PV>
__device__ __forceinline__ void load_vec(const T* ptr, float* o) {
  uint4 u;
  if constexpr (PV == 1) {
    u = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (sizeof(T) == 2) u.x = static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(ptr)) << 16;
    else u.x = __float_as_uint(*reinterpret_cast<const float*>(ptr));
  } else {
    u = *reinterpret_cast<const uint4*>(ptr);
  }
  TreeLoad<T, PV>::cvt(u, o);
}
template <typename T> __device__ __forceinline__ float logit_at(const T* row, int i) {
  float v;
  TreeLoad<T, 1>::cvt(TreeLoad<T, 1>::raw(row, i), &v);
  return v;
}

struct TreeShared {
  double tab[kExpTab];
  double xch[2][kTreeMaxCluster][4];   // per-CTA partials, double-buffered
  double red[kTreeWarps][4];           // per-warp partials
  float msm[kTreeWarps][2];            // per-warp online maxima
  double bc[4];                        // merged statistics, broadcast to the CTA
  double rcz[kMaxTreeNodes];           // residual chain: 1 / divisor of step j (float32 exponentials)
  int32_t cm[kMaxTreeNodes];           // residual chain: 1 residual, 0 renormalisation
  double rczx[kMaxTreeNodes];          // the same, exact (float64 exponentials), final node
  int32_t cmx[kMaxTreeNodes];
  int32_t par[kMaxTreeNodes];
  int32_t tok[kMaxTreeNodes];
  float ua[kMaxTreeNodes];
  float us[kMaxTreeNodes];
  int32_t drawn;
};

// Current distribution p' at one element: t, d the raw logits. Divisions by
// a pass's constants are multiplications by their reciprocals (one extra
// rounding each, far inside the draw's tie band).
struct NodeDist {
  double mt, md;           // row maxima (logit units)
  double rzt, rzd;         // reciprocals of the normalisers
  const double* rcz;       // residual chain: reciprocal of the divisor of step j
  const int32_t* cm;       // residual chain: 1 residual, 0 renormalisation
  int k;                   // residual steps taken at this node
};
__device__ __forceinline__ double ex64(const TreeShared& sm, double x) {
  return exp_fixup(x, exp_tbl(x, sm.tab), sm.tab);
}
__device__ __forceinline__ double p_at(const TreeShared& sm, const NodeDist& nd, double it, float t) {
  return ex64(sm, (t - nd.mt) * it) * nd.rzt;
}
__device__ __forceinline__ double q_at(const TreeShared& sm, const NodeDist& nd, double it, float d) {
  return ex64(sm, (d - nd.md) * it) * nd.rzd;
}
// p' after nd.k rejections, from p and q at the element
__device__ __forceinline__ double residual_chain(const NodeDist& nd, double a, double q) {
  for (int j = 0; j < nd.k; ++j) a = (nd.cm[j] ? fmax(a - q, 0.0) : a) * nd.rcz[j];
  return a;
}
// The same with float32 exponentials (c = log2(e) / T): statistics only.
__device__ __forceinline__ double p_cur32(const NodeDist& nd, float c, float t, float d, double* qv) {
  const double a = static_cast<double>(ex2((t - static_cast<float>(nd.mt)) * c)) * nd.rzt;
  const double q = static_cast<double>(ex2((d - static_cast<float>(nd.md)) * c)) * nd.rzd;
  *qv = q;
  return residual_chain(nd, a, q);
}

// Online maximum and sum of 2^((x - m) c) (M. Milakov and N. Gimelshein,
// "Online normalizer calculation for softmax", 2018) per thread: float32
// exponentials, a float32 sum with Kahan compensation (the sum is s - e).
struct OnlineSum {
  float m = -INFINITY, s = 0.f, e = 0.f;
};
template <int PV>
__device__ __forceinline__ void os_add(OnlineSum& o, const float* x, float c) {
  float vm = x[0];
#pragma unroll
  for (int k = 1; k < PV; ++k) vm = fmaxf(vm, x[k]);
  if (!(vm > -INFINITY)) return;
  if (vm > o.m) {
    const float f = o.m > -INFINITY ? ex2((o.m - vm) * c) : 0.f;
    o.s *= f;
    o.e *= f;
    o.m = vm;
  }
#pragma unroll
  for (int k = 0; k < PV; ++k) {
    const float y = ex2((x[k] - o.m) * c) - o.e;
    const float t = o.s + y;
    o.e = (t - o.s) - y;
    o.s = t;
  }
}
// Merge of per-lane (maximum, float64 sum) pairs over a warp: the maximum
// first, then every sum brought to it and added by a fixed butterfly.
__device__ __forceinline__ void ms_warp(float& m, double& s, float c) {
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  double v = (m > -INFINITY) ? s * static_cast<double>(ex2((m - M) * c)) : 0.0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  m = M;
  s = v;
}

// Block-wide sums of N values per thread into out[0..N): warp shuffles, then
// the warps in order.
template <int N>
__device__ void block_sum(TreeShared& sm, double* v, double* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < N; ++k)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < N; ++k) sm.red[warp][k] = v[k];
  __syncthreads();
  if (threadIdx.x < N) {
    double acc = sm.red[0][threadIdx.x];
    for (int w = 1; w < kTreeWarps; ++w) acc += sm.red[w][threadIdx.x];
    out[threadIdx.x] = acc;
  }
  __syncthreads();
}

// Every CTA's values cta[0..N) into every CTA's exchange buffer, then one
// cluster barrier; returns the buffer holding all ncl rows.
template <int N>
__device__ const double (*exchange(TreeShared& sm, const double* cta, int ncl, int& round))[4] {
  const int buf = round & 1;
  ++round;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x < ncl * N) {
    const int r = threadIdx.x / N, k = threadIdx.x - (threadIdx.x / N) * N;
    st_cluster_f64(&sm.xch[buf][rank][k], (uint32_t)r, cta[k]);
  }
  cluster_sync_all();
  return sm.xch[buf];
}
// Sums of the N exchanged values in rank order (identical in every CTA).
template <int N>
__device__ __forceinline__ void cluster_sum(const double (*x)[4], int ncl, double* out) {
#pragma unroll
  for (int k = 0; k < N; ++k) out[k] = x[0][k];
  for (int r = 1; r < ncl; ++r)
#pragma unroll
    for (int k = 0; k < N; ++k) out[k] += x[r][k];
}

template <typename T, int PV>
__global__ void __launch_bounds__(kTreeThreads, 1) tree_sample_kernel(const TreeParams p) {
  __shared__ TreeShared sm;
  __shared__ double cta[4];
  extern __shared__ __align__(128) unsigned char s_dyn[];   // staged slices: target, then draft
  __shared__ __align__(8) uint64_t s_bar;
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int rank = (int)cluster_ctarank();
  const int ncl = p.ncl;
  const int R = p.nodes, V = p.vocab;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this CTA's slice [beg, end), a multiple of PV * 32 wide except the last
  const int unit = PV * 32;
  const int chunk = ((V + ncl - 1) / ncl + unit - 1) / unit * unit;
  const int beg = min(V, rank * chunk), end = min(V, beg + chunk);
  const bool stage = p.stage != 0;
  const size_t stage_bytes = ((size_t)chunk * sizeof(T) + 127) / 128 * 128;
  T* s_t = reinterpret_cast<T*>(s_dyn);
  T* s_d = reinterpret_cast<T*>(s_dyn + stage_bytes);
  const uint32_t bar = smem_addr(&s_bar);
  uint32_t sphase = 0;
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  fill_exp_tab(sm.tab);
  for (int i = tid; i < R; i += kTreeThreads) {
    sm.par[i] = p.parents[(size_t)b * R + i];
    sm.tok[i] = p.tokens[(size_t)b * R + i];
    sm.ua[i] = p.u_accept[(size_t)b * R + i];
    sm.us[i] = p.u_sample[(size_t)b * R + i];
  }
  cluster_sync_all();                              // every CTA of the cluster runs; tables ready
  // a tree that breaks the parent rule is flagged and the walk draws at the root
  bool bad = sm.par[0] != -1;
  for (int c = 1; c < R; ++c) bad |= sm.par[c] < 0 || sm.par[c] >= c;
  if (bad && tid == 0 && rank == 0) flag_status(p.status, S3R_DEV_BAD_TREE);

  const double it = p.inv_temp;
  const float c32 = static_cast<float>(1.4426950408889634 * p.inv_temp);   // log2(e) / T
  constexpr int kStep = kTreeThreads * PV;
  int round = 0, v = 0, depth = 0;
  int32_t* out = p.out_tokens + (size_t)b * R;
  for (int guard = 0; guard < R; ++guard) {
    const T* tr = static_cast<const T*>(p.target) + ((size_t)b * R + v) * V;
    const T* dr = static_cast<const T*>(p.draft) + ((size_t)b * R + v) * V;
    bool has_child = false;
    for (int c = v + 1; c < R; ++c) has_child |= sm.par[c] == v;
    // the node's row slices: element i at tl[i - beg], dl[i - beg]
    const T* tl = tr + beg;
    const T* dl = dr + beg;
    if (stage) {
      fence_proxy_async_smem();                      // earlier reads of the buffers before the copies
      __syncthreads();
      if (tid == 0) {
        const uint32_t bytes = (uint32_t)(end - beg) * sizeof(T);
        mbar_arrive_expect_tx(bar, has_child ? 2u * bytes : bytes);
        for (uint32_t off = 0; off < bytes; off += kTreePiece) {
          const uint32_t sz = min(kTreePiece, bytes - off);
          bulk_load(smem_addr(s_t) + off, reinterpret_cast<const char*>(tl) + off, sz, bar);
          if (has_child) bulk_load(smem_addr(s_d) + off, reinterpret_cast<const char*>(dl) + off, sz, bar);
        }
      }
      mbar_wait(bar, sphase, nullptr, p.status);
      sphase ^= 1u;
      tl = s_t;
      dl = s_d;
    }
    // ---- one pass over the slices: row maxima (exact) and normalisers (float32
    // exponentials summed in float64), four vectors of each row in flight
    NodeDist nd;
    {
      OnlineSum ot, od;
      int i = beg + tid * PV;
      for (; i + 3 * kStep < end; i += 4 * kStep) {
        uint4 rt[4], rd[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) rt[u] = *reinterpret_cast<const uint4*>(tl + (i - beg) + u * kStep);
        if (has_child)
#pragma unroll
          for (int u = 0; u < 4; ++u) rd[u] = *reinterpret_cast<const uint4*>(dl + (i - beg) + u * kStep);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x[PV];
          TreeLoad<T, PV>::cvt(rt[u], x);
          os_add<PV>(ot, x, c32);
        }
        if (has_child)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float x[PV];
            TreeLoad<T, PV>::cvt(rd[u], x);
            os_add<PV>(od, x, c32);
          }
      }
      for (; i < end; i += kStep) {
        float x[PV];
        load_vec<T, PV>(tl + (i - beg), x);
        os_add<PV>(ot, x, c32);
        if (has_child) {
          load_vec<T, PV>(dl + (i - beg), x);
          os_add<PV>(od, x, c32);
        }
      }
      float mt = ot.m, md = od.m;
      double st = static_cast<double>(ot.s) - static_cast<double>(ot.e);
      double sd = static_cast<double>(od.s) - static_cast<double>(od.e);
      ms_warp(mt, st, c32);
      ms_warp(md, sd, c32);
      if (lane == 0) {
        sm.msm[warp][0] = mt;
        sm.msm[warp][1] = md;
        sm.red[warp][0] = st;
        sm.red[warp][1] = sd;
      }
      __syncthreads();
      if (warp == 0) {
        float m1 = lane < kTreeWarps ? sm.msm[lane][0] : -INFINITY, m2 = lane < kTreeWarps ? sm.msm[lane][1] : -INFINITY;
        double s1 = lane < kTreeWarps ? sm.red[lane][0] : 0.0, s2 = lane < kTreeWarps ? sm.red[lane][1] : 0.0;
        ms_warp(m1, s1, c32);
        ms_warp(m2, s2, c32);
        if (lane == 0) { cta[0] = m1; cta[1] = s1; cta[2] = m2; cta[3] = s2; }
      }
      __syncthreads();
      const double (*x)[4] = exchange<4>(sm, cta, ncl, round);
      if (warp == 0) {
        float m1 = lane < ncl ? static_cast<float>(x[lane][0]) : -INFINITY;
        float m2 = lane < ncl ? static_cast<float>(x[lane][2]) : -INFINITY;
        double s1 = lane < ncl ? x[lane][1] : 0.0, s2 = lane < ncl ? x[lane][3] : 0.0;
        ms_warp(m1, s1, c32);
        ms_warp(m2, s2, c32);
        if (lane == 0) { sm.bc[0] = m1; sm.bc[1] = s1; sm.bc[2] = m2; sm.bc[3] = s2; }
      }
      __syncthreads();
      nd.mt = sm.bc[0];
      nd.md = sm.bc[2];
      nd.rzt = 1.0 / sm.bc[1];
      nd.rzd = sm.bc[3] > 0.0 ? 1.0 / sm.bc[3] : 0.0;
    }
    nd.rcz = sm.rcz;
    nd.cm = sm.cm;
    nd.k = 0;
    // ---- the children in ascending order
    int next = -1;
    for (int c = v + 1; c < R && !bad; ++c) {
      if (sm.par[c] != v) continue;
      const int xc = sm.tok[c];
      double ratio = 0.0;
      if (xc >= 0 && xc < V) {
        const float tl = logit_at(tr, xc), dl = logit_at(dr, xc);
        const double qx = q_at(sm, nd, it, dl);
        ratio = qx > 0.0 ? residual_chain(nd, p_at(sm, nd, it, tl), qx) / qx : 0.0;
      } else if (tid == 0 && rank == 0) {
        flag_status(p.status, S3R_DEV_BAD_TOKEN_ID);
      }
      if (static_cast<double>(sm.ua[c]) < ratio) {
        next = c;
        break;
      }
      // rejected: p' <- max(p' - q, 0) / sum, or p' / sum(p') if that is all zero
      double s2[2] = {0.0, 0.0};
      for (int i = beg + tid * PV; i < end; i += kStep) {
        float xt[PV], xd[PV];
        load_vec<T, PV>(tl + (i - beg), xt);
        load_vec<T, PV>(dl + (i - beg), xd);
#pragma unroll
        for (int k = 0; k < PV; ++k) {
          double q;
          const double a = p_cur32(nd, c32, xt[k], xd[k], &q);
          s2[0] += fmax(a - q, 0.0);
          s2[1] += a;
        }
      }
      block_sum<2>(sm, s2, cta);
      double z[2];
      cluster_sum<2>(exchange<2>(sm, cta, ncl, round), ncl, z);
      // every thread has read the chain before this write (cluster barrier
      // in exchange()); nd.k < R <= kMaxTreeNodes
      if (tid == 0) {
        sm.cm[nd.k] = z[0] > 0.0 ? 1 : 0;
        sm.rcz[nd.k] = 1.0 / (z[0] > 0.0 ? z[0] : z[1]);
      }
      __syncthreads();
      ++nd.k;
    }
    if (next >= 0) {
      if (tid == 0 && rank == 0) {
        out[depth] = sm.tok[next];
        if (p.path) p.path[(size_t)b * R + depth] = next;
      }
      ++depth;
      v = next;
      continue;
    }
    // ---- the final node: exact weights for the draw
    NodeDist ndx = nd;
    // exact p and q of one vector; the PV exponentials are independent,
    // straight-line work
    auto exact_pq = [&](int i, double* pe, double* qe) {
      float xt[PV], xd[PV];
      load_vec<T, PV>(tl + (i - beg), xt);
      load_vec<T, PV>(dl + (i - beg), xd);
#pragma unroll
      for (int k = 0; k < PV; ++k) {
        pe[k] = p_at(sm, ndx, it, xt[k]);
        qe[k] = q_at(sm, ndx, it, xd[k]);
      }
    };
    if (nd.k == 0) {
      ndx.rzt = 1.0;                               // unnormalised exp((t - max) / T)
    } else {
      // normalisers with float64 exponentials, then the residual chain step
      // by step
      double z2[2] = {0.0, 0.0};
      for (int i = beg + tid * PV; i < end; i += kStep) {
        float xt[PV], xd[PV];
        load_vec<T, PV>(tl + (i - beg), xt);
        load_vec<T, PV>(dl + (i - beg), xd);
#pragma unroll
        for (int k = 0; k < PV; ++k) {
          z2[0] += ex64(sm, (xt[k] - nd.mt) * it);
          z2[1] += ex64(sm, (xd[k] - nd.md) * it);
        }
      }
      block_sum<2>(sm, z2, cta);
      double z[2];
      cluster_sum<2>(exchange<2>(sm, cta, ncl, round), ncl, z);
      ndx.rzt = 1.0 / z[0];
      ndx.rzd = 1.0 / z[1];
      ndx.rcz = sm.rczx;
      ndx.cm = sm.cmx;
      for (int j = 0; j < nd.k; ++j) {
        ndx.k = j;
        double zr[2] = {0.0, 0.0};
        for (int i = beg + tid * PV; i < end; i += kStep) {
          double pe[PV], qe[PV];
          exact_pq(i, pe, qe);
#pragma unroll
          for (int k = 0; k < PV; ++k) {
            const double a = residual_chain(ndx, pe[k], qe[k]);
            zr[0] += fmax(a - qe[k], 0.0);
            zr[1] += a;
          }
        }
        block_sum<2>(sm, zr, cta);
        double z[2];
        cluster_sum<2>(exchange<2>(sm, cta, ncl, round), ncl, z);
        if (tid == 0) {
          sm.cmx[j] = z[0] > 0.0 ? 1 : 0;
          sm.rczx[j] = 1.0 / (z[0] > 0.0 ? z[0] : z[1]);
        }
        __syncthreads();
      }
      ndx.k = nd.k;
    }
    // ---- draw from p' with u_sample[v]: every warp owns a contiguous
    // segment of the slice, walked in steps of 32 lanes x PV elements; a
    // lane's PV weights are summed in order, the lanes by an inclusive scan
    const int n = end - beg;
    const int seg = ((n + kTreeWarps - 1) / kTreeWarps + unit - 1) / unit * unit;
    const int w0 = beg + min(n, warp * seg), w1 = beg + min(n, (warp + 1) * seg);
    auto step_weights = [&](int s, double* w) {
      const int i = s + lane * PV;
      if (i < w1) {
        if (ndx.k == 0) {
          float xt[PV];
          load_vec<T, PV>(tl + (i - beg), xt);
#pragma unroll
          for (int k = 0; k < PV; ++k) w[k] = p_at(sm, ndx, it, xt[k]);
        } else {
          double pe[PV], qe[PV];
          exact_pq(i, pe, qe);
#pragma unroll
          for (int k = 0; k < PV; ++k) w[k] = residual_chain(ndx, pe[k], qe[k]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < PV; ++k) w[k] = 0.0;
      }
    };
    auto lane_scan = [&](double x) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      return x;
    };
    double run = 0.0;                                   // the warp's running sum
    int lastpos = -1;                                   // last positive-weight index of the warp
    for (int s = w0; s < w1; s += unit) {
      double w[PV], ls = 0.0;
      step_weights(s, w);
#pragma unroll
      for (int k = 0; k < PV; ++k) {
        ls += w[k];
        if (w[k] > 0.0) lastpos = s + lane * PV + k;
      }
      run += __shfl_sync(0xffffffffu, lane_scan(ls), 31);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lastpos = max(lastpos, __shfl_xor_sync(0xffffffffu, lastpos, o));
    if (lane == 0) {
      sm.red[warp][0] = run;
      sm.red[warp][1] = static_cast<double>(lastpos);
    }
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0, lp = -1.0;
      for (int w = 0; w < kTreeWarps; ++w) {
        tot += sm.red[w][0];
        lp = fmax(lp, sm.red[w][1]);
      }
      cta[0] = tot;
      cta[1] = lp;
    }
    __syncthreads();
    const double (*x)[4] = exchange<2>(sm, cta, ncl, round);
    double total = 0.0, lastall = -1.0;
    for (int r = 0; r < ncl; ++r) {
      total += x[r][0];
      lastall = fmax(lastall, x[r][1]);
    }
    const double thr = static_cast<double>(sm.us[v]) * total;
    // the CTA, then the warp, whose running sum first exceeds thr
    double pre = 0.0;
    int rsel = -1;
    for (int r = 0; r < ncl; ++r) {
      if (pre + x[r][0] > thr) { rsel = r; break; }
      pre += x[r][0];
    }
    if (tid == 0) sm.drawn = -1;
    __syncthreads();
    if (rsel == rank) {
      double wpre = pre;
      int wsel = -1;
      for (int w = 0; w < kTreeWarps; ++w) {
        if (wpre + sm.red[w][0] > thr) { wsel = w; break; }
        wpre += sm.red[w][0];
      }
      if (wsel == warp) {
        // the segment again, its running sum now started from the sums
        // before it; where rounding leaves no crossing, the segment's last
        // positive-weight index
        double run2 = wpre;
        int seg_last = -1;
        bool found = false;
        for (int s = w0; s < w1 && !found; s += unit) {
          double w[PV], ls = 0.0;
          step_weights(s, w);
#pragma unroll
          for (int k = 0; k < PV; ++k) {
            ls += w[k];
            if (w[k] > 0.0) seg_last = max(seg_last, s + lane * PV + k);
          }
          const double inc = lane_scan(ls);
          double exc = __shfl_up_sync(0xffffffffu, inc, 1);
          if (lane == 0) exc = 0.0;
          const unsigned hit = __ballot_sync(0xffffffffu, run2 + inc > thr);
          if (hit) {
            found = true;
            if (lane == __ffs(hit) - 1) {
              // the token inside this lane's PV weights
              double c = run2 + exc;
              int kk = -1, lastk = -1;
              for (int k = 0; k < PV; ++k) {
                c += w[k];
                if (w[k] > 0.0) lastk = k;
                if (c > thr) { kk = k; break; }
              }
              if (kk < 0) kk = lastk;                   // rounding inside the lane's sum
              sm.drawn = kk >= 0 ? s + lane * PV + kk : -1;
            }
          }
          run2 += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (!found) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) seg_last = max(seg_last, __shfl_xor_sync(0xffffffffu, seg_last, o));
          if (lane == 0) sm.drawn = seg_last;
        }
      }
    }
    __syncthreads();
    if (rsel == rank || (rsel < 0 && rank == 0)) {
      if (tid == 0) {
        // no crossing (rounding): the last index with positive weight
        const int tok = (rsel >= 0 && sm.drawn >= 0) ? sm.drawn : static_cast<int>(lastall);
        out[depth] = tok;
      }
    }
    break;
  }
  if (rank == 0 && tid == 0) {
    for (int i = depth + 1; i < R; ++i) out[i] = -1;
    if (p.path)
      for (int i = depth; i < R; ++i) p.path[(size_t)b * R + i] = -1;
    p.num_accepted[b] = depth;
  }
  cluster_sync_all();                                   // no CTA leaves while another may store into it
}

// Launch shapes already chosen in this process (the occupancy queries cost
// host time on every call otherwise), keyed by device, kernel, vocab size and
// sequence count. Only the choice is cached; nothing of a call's data.
struct TreeShape {
  int dev = -1, kern = -1, vocab = 0, nseq = 0, ncl = 0;
};
struct TreeShapeCache {
  std::mutex m;
  TreeShape e[16];
  int next = 0;
};
TreeShapeCache& tree_shapes() {
  static TreeShapeCache c;
  return c;
}

template <typename T, int PV>
cudaError_t launch_tree_typed(TreeParams p, cudaStream_t st) {
  auto kern = tree_sample_kernel<T, PV>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kTreeThreads);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  // the largest cluster (at most 8 CTAs) whose clusters all fit on the GPU
  // at once; when none does, 8. Rows 16-byte aligned (PV > 1) and slices
  // that fit: staged in shared memory.
  const int unit = PV * 32;
  auto stage_smem = [&](int c) -> size_t {
    if (PV == 1) return 0;
    const size_t chunk = (size_t)(((p.vocab + c - 1) / c + unit - 1) / unit * unit);
    const size_t bytes = 2 * ((chunk * sizeof(T) + 127) / 128 * 128);
    return bytes <= kTreeStageMax ? bytes : 0;
  };
  const int kid = (sizeof(T) == 2 ? 0 : 2) + (PV == 1 ? 0 : 1);
  int dev = 0;
  cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return ge;
  int pick = 0;
  {
    std::lock_guard<std::mutex> lk(tree_shapes().m);
    for (const TreeShape& t : tree_shapes().e)
      if (t.dev == dev && t.kern == kid && t.vocab == p.vocab && t.nseq == p.nseq) pick = t.ncl;
  }
  const int cmin = p.nseq * 2 <= 148 ? 2 : kTreeMaxCluster;      // more sequences: waves anyway
  for (int c = kTreeMaxCluster; pick == 0 && c >= cmin; --c) {
    const size_t smem = stage_smem(c);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(c, p.nseq);
    cfg.dynamicSmemBytes = smem;
    at[0].val.clusterDim.x = c;
    int nclusters = 0;
    cfg.numAttrs = 1;                                             // the cluster shape alone
    e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    cfg.numAttrs = 2;
    if (e != cudaSuccess) return e;
    if (nclusters >= p.nseq) pick = c;
  }
  if (pick == 0) pick = kTreeMaxCluster;
  {
    std::lock_guard<std::mutex> lk(tree_shapes().m);
    TreeShapeCache& tc = tree_shapes();
    bool known = false;
    for (const TreeShape& t : tc.e)
      known = known || (t.dev == dev && t.kern == kid && t.vocab == p.vocab && t.nseq == p.nseq);
    if (!known) {
      TreeShape& t = tc.e[tc.next];
      tc.next = (tc.next + 1) % 16;
      t.dev = dev; t.kern = kid; t.vocab = p.vocab; t.nseq = p.nseq; t.ncl = pick;
    }
  }
  const size_t pick_smem = stage_smem(pick);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pick_smem);
  if (e != cudaSuccess) return e;
  p.ncl = pick;
  p.stage = pick_smem > 0 ? 1 : 0;
  cfg.gridDim = dim3(pick, p.nseq);
  cfg.dynamicSmemBytes = pick_smem;
  at[0].val.clusterDim.x = pick;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

cudaError_t launch_tree_sample(const void* target, const void* draft, s3r_dtype dt, const int32_t* tokens,
                               const int32_t* parents, const float* u_accept, const float* u_sample, int32_t nseq,
                               int32_t nodes, int32_t vocab, double inv_temp, int32_t* out_tokens,
                               int32_t* num_accepted, int32_t* path, uint32_t* status, bool vec, cudaStream_t st) {
  TreeParams p{};
  p.target = target;
  p.draft = draft;
  p.tokens = tokens;
  p.parents = parents;
  p.u_accept = u_accept;
  p.u_sample = u_sample;
  p.out_tokens = out_tokens;
  p.num_accepted = num_accepted;
  p.path = path;
  p.nseq = nseq;
  p.nodes = nodes;
  p.vocab = vocab;
  p.inv_temp = inv_temp;
  p.status = status;
  if (dt == S3R_BF16)
    return vec ? launch_tree_typed<__nv_bfloat16, 8>(p, st) : launch_tree_typed<__nv_bfloat16, 1>(p, st);
  return vec ? launch_tree_typed<float, 4>(p, st) : launch_tree_typed<float, 1>(p, st);
}

}  // namespace s3r
