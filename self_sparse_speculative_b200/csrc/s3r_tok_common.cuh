// Pieces shared by the token-major tcgen05 attention kernels (the dense /
// split-KV kernel in s3r_attn_tok.cu and the fused sparse draft kernel in
// s3r_draft_fused.cu): the shared-memory layout of Q, P and the K/V ring, and
// the row-wise reductions of the softmax warpgroup.
#pragma once

#include <cuda_bf16.h>

#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {

constexpr int kTok = 128;                    // tokens per stage (MMA M of S^T)
constexpr float kTau = 8.0f;                 // lazy reference slack, log2 units
constexpr float kNuInit = 1e30f;             // -(reference) before the first score of a segment
constexpr int kTokSmemBudget = 232448 - 8192;
constexpr int kMaxPend = 8;                  // deferred split-unit combines per CTA

template <int N, int D>
struct TokLay {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQBytes = N * D * 2;           // [d half][N rows][128 B]
  static constexpr uint32_t kPBytes = N * kTok * 2;        // [token half][N rows][128 B]
  static constexpr uint32_t kTileBytes = kTok * D * 2;     // K or V of one stage: [d half][128 tokens][128 B]
  static constexpr int kNSraw = (kTokSmemBudget - (int)kQBytes - (int)kPBytes) / (2 * (int)kTileBytes);
  static constexpr int kNS = kNSraw > 6 ? 6 : kNSraw;
  // two P buffers (softmax(g) then waits only for PV(g - 2)) when they fit
  // without losing a stage
  static constexpr int kPBufs =
      (kTokSmemBudget - (int)kQBytes - 2 * (int)kPBytes) / (2 * (int)kTileBytes) >= kNS ? 2 : 1;
  static constexpr uint32_t kOffP = kQBytes;
  static constexpr uint32_t kOffKV = kOffP + kPBufs * kPBytes;
  static constexpr uint32_t kDynBytes = kOffKV + kNS * 2 * kTileBytes;
  static constexpr uint32_t kColS = 0, kColO = 2 * N;      // S^T[2], O^T
  static constexpr int kQChunks = N * D / 8 / 128;         // 16-byte Q chunks per softmax thread
  static_assert(kNS >= 2, "pipeline needs two stages");
  static_assert(3 * N <= 256, "TMEM columns");
};

// Reduce N per-thread values per row over the warp: afterwards lane l holds
// the result for row l of v[0..C) (C = 32), or row l % 16 (C = 16).
template <int C, bool kMax>
__device__ __forceinline__ float warp_rows_reduce(float* v, int lane) {
#pragma unroll
  for (int w = C / 2; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int k = 0; k < w; ++k) {
      const float send = up ? v[k] : v[k + w];
      const float keep = up ? v[k + w] : v[k];
      const float got = __shfl_xor_sync(0xffffffffu, send, w);
      v[k] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = C; o < 32; o <<= 1) {                  // lanes that hold the same row
    const float x = __shfl_xor_sync(0xffffffffu, r, o);
    r = kMax ? fmaxf(r, x) : r + x;
  }
  return r;
}

// Row-wise reduction over the 128 softmax threads into red[row] (N rows).
template <int N, bool kMax>
__device__ __forceinline__ void wg_rows_reduce(float* v, float (*s_red)[64], float* out, int q4, int lane,
                                               int tid) {
#pragma unroll
  for (int c0 = 0; c0 < N; c0 += 32) {
    if (N - c0 >= 32) {
      const float r = warp_rows_reduce<32, kMax>(v + c0, lane);
      s_red[q4][c0 + lane] = r;
    } else if (N - c0 >= 16) {
      const float r = warp_rows_reduce<16, kMax>(v + c0, lane);
      if (lane < 16) s_red[q4][c0 + lane] = r;
      if (N - c0 > 16) {
        const float r8 = warp_rows_reduce<8, kMax>(v + c0 + 16, lane);
        if (lane < 8) s_red[q4][c0 + 16 + lane] = r8;
      }
    } else {
      const float r = warp_rows_reduce<8, kMax>(v + c0, lane);
      if (lane < 8) s_red[q4][c0 + lane] = r;
    }
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (tid < N) {
    const float a = s_red[0][tid], b = s_red[1][tid], c = s_red[2][tid], d = s_red[3][tid];
    out[tid] = kMax ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
  }
}

// Number of the 128 softmax threads whose predicate is true (named barrier 1).
__device__ __forceinline__ int wg_count(bool pred) {
  int r;
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.popc.u32 %0, 1, 128, p;\n\t}"
               : "=r"(r) : "r"((int)pred) : "memory");
  return r;
}

}  // namespace s3r
