// Pieces shared by the bf16 (tensor-core) and fp32 attention kernels: output
// addressing, the log-sum-exp merge of split partials, and empty outputs.
#pragma once

#include <cuda_bf16.h>

#include <cmath>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {

constexpr float kLn2 = 0.6931471805599453f;

template <typename OutT>
__device__ __forceinline__ void store_out4(OutT* dst, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store_out4<__nv_bfloat16>(__nv_bfloat16* dst, float a, float b, float c, float d) {
  uint2 v = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
  *reinterpret_cast<uint2*>(dst) = v;
}
template <>
__device__ __forceinline__ void store_out4<float>(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}

// Packed row i of unit (b, h) is query head h*G + (i % G) of verify row i / G;
// its output row in the [S, R, Hq] layout.
__device__ __forceinline__ size_t out_row_offset(const AttnParams& p, int b, int h, int i) {
  const int r = i / p.G, g = i - (i / p.G) * p.G;
  return ((size_t)(b * p.R + r) * p.Hq + (size_t)h * p.G + g);
}

// Merge partial states slots [slot0, slot0 + nparts) of unit (b, h) into the
// final output: M = max m_s, L = sum l_s 2^(m_s - M), out = sum O_s 2^(m_s - M) / L,
// lse = (M + log2 L) ln 2 (m in log2 units of the scaled score).
// Runs on threads [0, nthreads) of the CTA; partials are read through L2.
template <typename OutT>
__device__ void combine_partials(const AttnParams& p, int b, int h, int slot0, int nparts, int nthreads) {
  const int D4 = p.D / 4;
  for (int idx = threadIdx.x; idx < p.rows * D4; idx += nthreads) {
    const int i = idx / D4, d4 = idx - (idx / D4) * D4;
    float M = -INFINITY;
    for (int s = 0; s < nparts; ++s) {
      const float m = __ldcg(p.part_ml + ((size_t)(slot0 + s) * p.rows + i) * 2);
      M = fmaxf(M, m);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float Ls = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < nparts; ++s) {
        const size_t pi = (size_t)(slot0 + s) * p.rows + i;
        const float m = __ldcg(p.part_ml + pi * 2), l = __ldcg(p.part_ml + pi * 2 + 1);
        if (m == -INFINITY || l == 0.f) continue;
        const float w = exp2f(m - M);
        Ls += l * w;
        const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + pi * p.D) + d4);
        acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    const size_t orow = out_row_offset(p, b, h, i);
    store_out4<OutT>(static_cast<OutT*>(p.out) + orow * p.D + d4 * 4, acc.x * inv, acc.y * inv, acc.z * inv,
                     acc.w * inv);
    if (d4 == 0 && p.lse) p.lse[orow] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
  }
}

// Outputs of a unit whose context length is invalid: zeros and lse = -inf.
template <typename OutT>
__device__ void write_empty_unit(const AttnParams& p, int b, int h, int tid0, int nthreads) {
  const int D4 = p.D / 4;
  for (int idx = tid0; idx < p.rows * D4; idx += nthreads) {
    const int i = idx / D4, d4 = idx - (idx / D4) * D4;
    const size_t orow = out_row_offset(p, b, h, i);
    store_out4<OutT>(static_cast<OutT*>(p.out) + orow * p.D + d4 * 4, 0.f, 0.f, 0.f, 0.f);
    if (d4 == 0 && p.lse) p.lse[orow] = -INFINITY;
  }
}

// Whether sequence b's context length is usable for `R` query rows.
__device__ __forceinline__ bool bad_context(const AttnParams& p, int L) {
  return L < p.R || L < 1 || L > p.max_pages * p.P;
}

// Pages one KV head of sequence b attends over: all n_b pages (verify) or
// min(budget, n_b) selected pages (draft); 0 for an unusable length.
__device__ __forceinline__ int unit_pages(const AttnParams& p, int L) {
  if (bad_context(p, L)) return 0;
  const int n_b = (L + p.P - 1) / p.P;
  return p.page_list ? min(p.budget, n_b) : n_b;
}

}  // namespace s3r
