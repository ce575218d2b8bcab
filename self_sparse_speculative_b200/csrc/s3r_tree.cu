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
// One thread-block cluster of kTreeCluster CTAs per sequence; CTA r owns the
// vocab slice r. The walk is sequential, each of its vocab-wide quantities a
// pass over the slices whose per-CTA results every CTA stores into every
// other CTA's shared memory (st.shared::cluster) before a cluster barrier;
// every CTA then combines them in rank order, so all of them hold identical
// values and take identical decisions without another round trip. The first
// pass over a node's rows reads HBM, the later ones hit L2. Sums and
// normalisers are float64 with table-driven exponentials (exp_tbl).
#include <cuda_bf16.h>

#include <cmath>

#include "s3r_device.cuh"
#include "s3r_exp64.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kTreeThreads = 512;
constexpr int kTreeWarps = kTreeThreads / 32;
constexpr int kTreeCluster = 8;

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
  double inv_temp;
  uint32_t* status;
};

// PV logits from element i of a row (PV > 1: i a multiple of PV, the row
// 16-byte aligned).
template <typename T, int PV> struct TreeLoad;
template <> struct TreeLoad<__nv_bfloat16, 8> {
  static __device__ __forceinline__ void at(const __nv_bfloat16* row, int i, float* o) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + i));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = __uint_as_float(w[k] << 16);
      o[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};
template <> struct TreeLoad<float, 4> {
  static __device__ __forceinline__ void at(const float* row, int i, float* o) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(row + i));
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
};
template <typename T> struct TreeLoad<T, 1> {
  static __device__ __forceinline__ void at(const T* row, int i, float* o) {
    if constexpr (sizeof(T) == 2) o[0] = __bfloat162float(row[i]);
    else o[0] = row[i];
  }
};
template <typename T> __device__ __forceinline__ float logit_at(const T* row, int i) {
  float v;
  TreeLoad<T, 1>::at(row, i, &v);
  return v;
}

struct TreeShared {
  double tab[kExpTab];
  double xch[2][kTreeCluster][4];    // per-CTA partials, double-buffered
  double red[kTreeWarps][4];         // per-warp partials
  double cz[kMaxTreeNodes];          // residual chain: divisor of step j
  int32_t cm[kMaxTreeNodes];         // residual chain: 1 residual, 0 renormalisation
  int32_t par[kMaxTreeNodes];
  int32_t tok[kMaxTreeNodes];
  float ua[kMaxTreeNodes];
  float us[kMaxTreeNodes];
  int32_t drawn;
};

// Current distribution p' at one element: t, d the raw logits.
struct NodeDist {
  double mt, md, zt, zd;   // row maxima (logit units) and normalisers
  int k;                   // residual steps taken at this node
};
__device__ __forceinline__ double ex64(const TreeShared& sm, double x) {
  return exp_fixup(x, exp_tbl(x, sm.tab), sm.tab);
}
__device__ __forceinline__ double p_at(const TreeShared& sm, const NodeDist& nd, double it, float t) {
  return ex64(sm, (t - nd.mt) * it) / nd.zt;
}
__device__ __forceinline__ double q_at(const TreeShared& sm, const NodeDist& nd, double it, float d) {
  return ex64(sm, (d - nd.md) * it) / nd.zd;
}
// p' after nd.k rejections, from p and q at the element
__device__ __forceinline__ double residual_chain(const TreeShared& sm, int k, double a, double q) {
  for (int j = 0; j < k; ++j) a = sm.cm[j] ? fmax(a - q, 0.0) / sm.cz[j] : a / sm.cz[j];
  return a;
}
__device__ __forceinline__ double p_cur(const TreeShared& sm, const NodeDist& nd, double it, float t, float d) {
  const double a = p_at(sm, nd, it, t);
  return nd.k == 0 ? a : residual_chain(sm, nd.k, a, q_at(sm, nd, it, d));
}

// Block-wide sums (or maxima) of n values per thread into out[0..n): warp
// shuffles, then warp 0 over the warps in order.
template <int N, bool MAX>
__device__ void block_reduce(TreeShared& sm, double* v, double* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < N; ++k)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double w = __shfl_xor_sync(0xffffffffu, v[k], o);
      v[k] = MAX ? fmax(v[k], w) : v[k] + w;
    }
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < N; ++k) sm.red[warp][k] = v[k];
  __syncthreads();
  if (threadIdx.x < N) {
    double acc = sm.red[0][threadIdx.x];
    for (int w = 1; w < kTreeWarps; ++w) acc = MAX ? fmax(acc, sm.red[w][threadIdx.x]) : acc + sm.red[w][threadIdx.x];
    out[threadIdx.x] = acc;
  }
  __syncthreads();
}

// Every CTA's values cta[0..n) into every CTA's exchange buffer, then one
// cluster barrier; returns the buffer holding all kTreeCluster rows.
template <int N>
__device__ const double (*exchange(TreeShared& sm, const double* cta, int& round))[4] {
  const int buf = round & 1;
  ++round;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x < kTreeCluster * N) {
    const int r = threadIdx.x / N, k = threadIdx.x - (threadIdx.x / N) * N;
    st_cluster_f64(&sm.xch[buf][rank][k], (uint32_t)r, cta[k]);
  }
  cluster_sync_all();
  return sm.xch[buf];
}

template <typename T, int PV>
__global__ void __launch_bounds__(kTreeThreads, 1) tree_sample_kernel(const TreeParams p) {
  __shared__ TreeShared sm;
  __shared__ double cta[4];
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int rank = (int)cluster_ctarank();
  const int R = p.nodes, V = p.vocab;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this CTA's slice [beg, end), a multiple of PV * 32 wide except the last
  const int unit = PV * 32;
  const int chunk = ((V + kTreeCluster - 1) / kTreeCluster + unit - 1) / unit * unit;
  const int beg = min(V, rank * chunk), end = min(V, beg + chunk);
  fill_exp_tab(sm.tab);
  for (int i = tid; i < R; i += kTreeThreads) {
    sm.par[i] = p.parents[(size_t)b * R + i];
    sm.tok[i] = p.tokens[(size_t)b * R + i];
    sm.ua[i] = p.u_accept[(size_t)b * R + i];
    sm.us[i] = p.u_sample[(size_t)b * R + i];
  }
  cluster_sync_all();                                   // every CTA of the cluster runs; tables ready
  // a tree that breaks the parent rule is flagged and cut where it breaks
  bool bad = sm.par[0] != -1;
  for (int c = 1; c < R; ++c) bad |= sm.par[c] < 0 || sm.par[c] >= c;
  if (bad && tid == 0 && rank == 0) flag_status(p.status, S3R_DEV_BAD_TREE);

  const double it = p.inv_temp;
  int round = 0, v = 0, depth = 0;
  int32_t* out = p.out_tokens + (size_t)b * R;
  for (int guard = 0; guard < R; ++guard) {
    const T* tr = static_cast<const T*>(p.target) + ((size_t)b * R + v) * V;
    const T* dr = static_cast<const T*>(p.draft) + ((size_t)b * R + v) * V;
    bool has_child = false;
    for (int c = v + 1; c < R; ++c) has_child |= sm.par[c] == v;
    // ---- row maxima (exact in float)
    NodeDist nd;
    {
      float mt = -INFINITY, md = -INFINITY;
      for (int i = beg + tid * PV; i < end; i += kTreeThreads * PV) {
        float x[PV];
        TreeLoad<T, PV>::at(tr, i, x);
#pragma unroll
        for (int k = 0; k < PV; ++k) mt = fmaxf(mt, x[k]);
        if (has_child) {
          TreeLoad<T, PV>::at(dr, i, x);
#pragma unroll
          for (int k = 0; k < PV; ++k) md = fmaxf(md, x[k]);
        }
      }
      double m2[2] = {mt, md};
      block_reduce<2, true>(sm, m2, cta);
      const double (*x)[4] = exchange<2>(sm, cta, round);
      nd.mt = x[0][0];
      nd.md = x[0][1];
      for (int r = 1; r < kTreeCluster; ++r) {
        nd.mt = fmax(nd.mt, x[r][0]);
        nd.md = fmax(nd.md, x[r][1]);
      }
    }
    // ---- normalisers
    {
      double zt = 0.0, zd = 0.0;
      for (int i = beg + tid * PV; i < end; i += kTreeThreads * PV) {
        float x[PV];
        TreeLoad<T, PV>::at(tr, i, x);
#pragma unroll
        for (int k = 0; k < PV; ++k) {
          const double e = (x[k] - nd.mt) * it;
          zt += exp_fixup(e, exp_tbl(e, sm.tab), sm.tab);
        }
        if (has_child) {
          TreeLoad<T, PV>::at(dr, i, x);
#pragma unroll
          for (int k = 0; k < PV; ++k) {
            const double e = (x[k] - nd.md) * it;
            zd += exp_fixup(e, exp_tbl(e, sm.tab), sm.tab);
          }
        }
      }
      double z2[2] = {zt, zd};
      block_reduce<2, false>(sm, z2, cta);
      const double (*x)[4] = exchange<2>(sm, cta, round);
      nd.zt = x[0][0];
      nd.zd = x[0][1];
      for (int r = 1; r < kTreeCluster; ++r) {
        nd.zt += x[r][0];
        nd.zd += x[r][1];
      }
    }
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
        ratio = qx > 0.0 ? residual_chain(sm, nd.k, p_at(sm, nd, it, tl), qx) / qx : 0.0;
      } else if (tid == 0 && rank == 0) {
        flag_status(p.status, S3R_DEV_BAD_TOKEN_ID);
      }
      if (static_cast<double>(sm.ua[c]) < ratio) {
        next = c;
        break;
      }
      // rejected: p' <- max(p' - q, 0) / sum, or p' / sum(p') if that is all zero
      double s2[2] = {0.0, 0.0};
      for (int i = beg + tid * PV; i < end; i += kTreeThreads * PV) {
        float xt[PV], xd[PV];
        TreeLoad<T, PV>::at(tr, i, xt);
        TreeLoad<T, PV>::at(dr, i, xd);
#pragma unroll
        for (int k = 0; k < PV; ++k) {
          const double q = q_at(sm, nd, it, xd[k]);
          const double a = residual_chain(sm, nd.k, p_at(sm, nd, it, xt[k]), q);
          s2[0] += fmax(a - q, 0.0);
          s2[1] += a;
        }
      }
      block_reduce<2, false>(sm, s2, cta);
      const double (*x)[4] = exchange<2>(sm, cta, round);
      double zr = x[0][0], za = x[0][1];
      for (int r = 1; r < kTreeCluster; ++r) {
        zr += x[r][0];
        za += x[r][1];
      }
      if (nd.k < kMaxTreeNodes) {                   // nd.k < R <= kMaxTreeNodes always
        // every thread has read the chain (p_cur above) before this write:
        // the cluster barrier in exchange() sits between
        if (tid == 0) {
          sm.cm[nd.k] = zr > 0.0 ? 1 : 0;
          sm.cz[nd.k] = zr > 0.0 ? zr : za;
        }
        __syncthreads();
        ++nd.k;
      }
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
    // ---- draw from p' with u_sample[v]: every warp owns a contiguous
    // segment of the slice, walked in steps of 32 lanes x PV elements; a
    // lane's PV weights are summed in order, the lanes by an inclusive scan
    const int n = end - beg;
    const int seg = ((n + kTreeWarps - 1) / kTreeWarps + unit - 1) / unit * unit;
    const int w0 = beg + min(n, warp * seg), w1 = beg + min(n, (warp + 1) * seg);
    auto step_weights = [&](int s, double* w) {
      const int i = s + lane * PV;
      if (i < w1) {
        float xt[PV], xd[PV];
        TreeLoad<T, PV>::at(tr, i, xt);
        if (nd.k > 0) TreeLoad<T, PV>::at(dr, i, xd);
#pragma unroll
        for (int k = 0; k < PV; ++k) w[k] = p_cur(sm, nd, it, xt[k], nd.k > 0 ? xd[k] : 0.f);
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
    const double (*x)[4] = exchange<2>(sm, cta, round);
    double total = 0.0, lastall = -1.0;
    for (int r = 0; r < kTreeCluster; ++r) {
      total += x[r][0];
      lastall = fmax(lastall, x[r][1]);
    }
    const double thr = static_cast<double>(sm.us[v]) * total;
    // the CTA, then the warp, whose running sum first exceeds thr
    double pre = 0.0;
    int rsel = -1;
    for (int r = 0; r < kTreeCluster; ++r) {
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

template <typename T, int PV>
cudaError_t launch_tree_typed(const TreeParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kTreeCluster, p.nseq);
  cfg.blockDim = dim3(kTreeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kTreeCluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tree_sample_kernel<T, PV>, p);
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
