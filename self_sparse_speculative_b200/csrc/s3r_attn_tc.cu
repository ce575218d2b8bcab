// Persistent tensor-core (tcgen05) split-KV paged attention, bf16, for the
// S3R sparse draft and dense verify steps ("S3R: Fast and Faithful RL
// Rollouts via Self-Sparse Speculative Decoding", weekinpapers.com,
// Abstract: sparse attention proposes, full attention over the complete KV
// history verifies, both over one shared cache).
//
// Work partition (stream-K style). The work is the flattened list of
// (sequence, KV head, page) triples: all n_b pages of every KV head (verify)
// or the min(B, n_b) selected pages (draft). Every CTA (one per SM) takes one
// contiguous range of W = ceil(total / grid) of them, so the load is even to
// within one page whatever the context lengths. A range crosses (sequence,
// KV head) units; each maximal piece of one unit is a "segment" with its own
// softmax state. A unit split over several CTAs is merged by log-sum-exp in
// the epilogue of the last of them to finish (atomic ticket, no waiting).
//
// Per segment the G query heads x R rows of the unit are packed into the rows
// of one MMA tile (M = 64, or 128 above 64 rows), so every 64-token K/V tile
// read from HBM feeds one dense contraction:
//   S = Q K^T (M x 64, K = D) and O += P V (M x D, K = 64), fp32 in TMEM.
// Warp roles (320 threads):
//   warps 0-7  two softmax warpgroups working on alternate stages (ping-pong),
//              each with its own S, P and O buffers; warpgroup 0 also merges
//              the two partial states and writes each segment's output;
//   warp 8     producer: resolves page ids ahead of use, loads each segment's
//              Q into a double buffer, prefetches K/V tiles 8 stages ahead
//              into L2 and streams them by TMA (3-D tensor map, 128-byte
//              swizzle) into an NS-stage ring;
//   warp 9     MMA issuer (one thread, QK two stages ahead of PV) and TMEM
//              owner.
// TMEM: S[2] (64 columns each) and O[2] (D columns each), one per stream.
// The running max is rescaled lazily (only when it grows by more than 2^8);
// O and l always share one reference, so the result is exact.
#include <cuda_bf16.h>

#include <cmath>

#include "s3r_attn_common.cuh"
#include "s3r_attn_sched.cuh"
#include "s3r_device.cuh"
#include "s3r_internal.h"

namespace s3r {
namespace {

constexpr int kThreads = 320;               // 2 softmax warpgroups + producer + MMA
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleTau = 8.0f;      // log2 units
constexpr int kSmemBudget = 232448 - 8192;

template <int M, int D>
struct Lay {
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQBytes = M * D * 2;
  static constexpr uint32_t kPBytes = M * 128;
  static constexpr uint32_t kTileBytes = kStageTokens * D * 2;       // K or V of one stage
  static constexpr int kNSraw = (kSmemBudget - 2 * (int)kQBytes - 2 * (int)kPBytes) / (2 * (int)kTileBytes);
  static constexpr int kNS = kNSraw > 8 ? 8 : kNSraw;
  static constexpr uint32_t kOffP = 2 * kQBytes;
  static constexpr uint32_t kOffKV = kOffP + 2 * kPBytes;
  static constexpr uint32_t kDynBytes = kOffKV + kNS * 2 * kTileBytes;
  static constexpr uint32_t kColS = 0, kColO = 2 * kStageTokens;
  static constexpr uint32_t kTmemCols = (kColO + 2 * D) <= 256 ? 256 : 512;
  static_assert(kNS >= 2, "pipeline needs two stages");
};

template <int M, int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const AttnParams p) {
  using L = Lay<M, D>;
  constexpr int NS = L::kNS;
  extern __shared__ __align__(1024) uint8_t dyn_raw[];
  uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t s_bar[2 * NS + 14];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_ticket;
  __shared__ int s_prefix[kMaxSeqs + 1];
  __shared__ int s_stage_lp[NS][4];
  __shared__ float s_ml[2][2][128];                      // [segment parity][m, l][row] of stream 1

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();

  // ---- per-sequence prefix of unit pages (warp 0), range of this CTA
  if (warp == 0) {
    const int per = (p.S + 31) / 32;
    const int b0 = min(p.S, lane * per), b1 = min(p.S, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) sum += unit_pages(p, p.context_lens[b]) * p.Hkv;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
    for (int b = b0; b < b1; ++b) {
      s_prefix[b] = run;
      run += unit_pages(p, p.context_lens[b]) * p.Hkv;
    }
    if (lane == 31) s_prefix[p.S] = incl;
  }
  __syncthreads();
  pdl_wait();                                           // earlier kernels' results are visible from here
  if (blockIdx.x == 0) {
    // unusable lengths: flag them, give their rows zero output and lse -inf
    for (int b = 0; b < p.S; ++b) {
      if (!bad_context(p, p.context_lens[b])) continue;
      if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
      for (int h = 0; h < p.Hkv; ++h) write_empty_unit<__nv_bfloat16>(p, b, h, tid, kThreads);
    }
  }
  const int total = s_prefix[p.S];
  const int W = (total + gridDim.x - 1) / gridDim.x;
  const int lo = blockIdx.x * W, hi = min(total, lo + W);
  if (lo >= hi) return;                                 // uniform over the CTA
  const int ppt = kStageTokens / p.P;

  // ---- barriers
  const uint32_t bar0 = smem_addr(&s_bar[0]);
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const int B_FULL = 0, B_EMPTY = NS, B_SFULL = 2 * NS, B_PFULL = 2 * NS + 2, B_ODONE = 2 * NS + 4,
            B_OFULL = 2 * NS + 6, B_OEMPTY = 2 * NS + 8, B_QFULL = 2 * NS + 9, B_QEMPTY = 2 * NS + 11,
            B_TD = 2 * NS + 13;
  uint8_t* sP = dyn + L::kOffP;
  uint8_t* sKV = dyn + L::kOffKV;
  const uint32_t aQ = smem_addr(dyn), aP = smem_addr(sP), aKV = smem_addr(sKV);

  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(&s_tmem), L::kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(BAR(B_FULL + i), 1); mbar_init(BAR(B_EMPTY + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(B_SFULL + i), 1);
      mbar_init(BAR(B_PFULL + i), 128);
      mbar_init(BAR(B_ODONE + i), 1);
      mbar_init(BAR(B_OFULL + i), 1);
      mbar_init(BAR(B_QFULL + i), 32);
      mbar_init(BAR(B_QEMPTY + i), 1);
    }
    mbar_init(BAR(B_OEMPTY), 128);
    mbar_init(BAR(B_TD), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) { prefetch_tensormap(&tmK); prefetch_tensormap(&tmV); }
  // zero both Q buffers (padding rows stay zero) and both P buffers
  for (int i = tid; i < (int)((2 * L::kQBytes + 2 * L::kPBytes) / 16); i += kThreads)
    reinterpret_cast<uint4*>(dyn)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == kProducerWarp) {
    // ======================================================= producer warp
    const uint64_t pol = l2_policy_evict_first();
    // page-id windows of 32 flattened positions: lane k of a window holds
    // position wbase + k. w0 = in use, w1 = phys loads in flight, w2 = lp
    // loads in flight.
    int w0_lp, w0_ph, w0_u, w1_lp, w1_ph, w1_u, w2_lp, w2_u;
    // issue the block-table load of a page (checked against the sequence
    // length first; the loaded id is range-checked where it is used)
    auto phys_load = [&](int lp, int u) {
      if (lp < 0) return -1;
      const int b = u / p.Hkv;
      const int n_b = (p.context_lens[b] + p.P - 1) / p.P;
      if (lp >= n_b) { flag_status(p.status, S3R_DEV_BAD_PAGE_ID); return -1; }
      return p.block_table[(size_t)b * p.max_pages + lp];
    };
    int wbase = lo;
    page_of(p, s_prefix, wbase + lane, hi, W, &w0_lp, &w0_u);
    w0_ph = phys_load(w0_lp, w0_u);
    page_of(p, s_prefix, wbase + 32 + lane, hi, W, &w1_lp, &w1_u);
    w1_ph = phys_load(w1_lp, w1_u);
    page_of(p, s_prefix, wbase + 64 + lane, hi, W, &w2_lp, &w2_u);
    // L2 prefetch distance in flattened positions (8 stages ahead, <= 32)
    const int pfd = 8 * ppt;
    int g = 0;
    bool ok = true;
    int s = 0;
    for (int x = lo; x < hi && ok; ++s) {
      const Seg sg = locate(p, s_prefix, x, hi, W);
      // Q of this segment -> Q[s & 1] (rows in order, K-major 128-byte swizzle)
      if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_QEMPTY + (s & 1)), ((s >> 1) & 1) ^ 1, &s_abort, p.status))) {
        ok = false;
        break;
      }
      {
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
        uint8_t* sQ = dyn + (s & 1) * L::kQBytes;
        constexpr int kChunks = D / 8;
        for (int c = lane; c < p.rows * kChunks; c += 32) {
          const int i = c / kChunks, c16 = c - (c / kChunks) * kChunks;
          const uint4 v = *reinterpret_cast<const uint4*>(q + out_row_offset(p, sg.b, sg.h, i) * D + c16 * 8);
          *reinterpret_cast<uint4*>(sQ + (c16 >> 3) * (M * 128) + i * 128 + (((c16 & 7) ^ (i & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        mbar_arrive(BAR(B_QFULL + (s & 1)));
      }
      const int nst = (sg.npg + ppt - 1) / ppt;
      for (int j = 0; j < nst; ++j, ++g) {
        const int st = g % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_EMPTY + st), ((g / NS) & 1) ^ 1, &s_abort, p.status))) {
          ok = false;
          break;
        }
        // page ids of this stage: positions x + j*ppt + pp (pp < ppt)
        int my_lp = -1, my_ph = -1, pf_z = -1;
        for (int pp = 0; pp < ppt; ++pp) {
          // positions past the segment belong to the next one: the windows
          // must not move past its first page (warp-uniform)
          if (j * ppt + pp >= sg.npg) break;
          const int xp = x + j * ppt + pp;
          while (xp >= wbase + 32) {                   // advance the windows (warp-uniform)
            wbase += 32;
            w0_lp = w1_lp; w0_ph = w1_ph; w0_u = w1_u;
            w1_lp = w2_lp; w1_u = w2_u;
            w1_ph = phys_load(w1_lp, w1_u);
            page_of(p, s_prefix, wbase + 64 + lane, hi, W, &w2_lp, &w2_u);
          }
          const int src = xp - wbase;
          const int lp = __shfl_sync(0xffffffffu, w0_lp, src & 31);
          int ph = __shfl_sync(0xffffffffu, w0_ph, src & 31);
          if (lp >= 0 && (ph < 0 || ph >= p.num_pages_total)) {
            if (lane == 0) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
            ph = -1;
          }
          if (lane == pp) { my_lp = lp; my_ph = ph; }
          // the page pfd positions ahead, into L2 (whatever unit it belongs to)
          const int s2 = src + pfd;
          const int lp2 = __shfl_sync(0xffffffffu, s2 < 32 ? w0_lp : w1_lp, s2 & 31);
          const int ph2 = __shfl_sync(0xffffffffu, s2 < 32 ? w0_ph : w1_ph, s2 & 31);
          const int u2 = __shfl_sync(0xffffffffu, s2 < 32 ? w0_u : w1_u, s2 & 31);
          if (lane == pp && xp + pfd < hi && lp2 >= 0 && ph2 >= 0 && ph2 < p.num_pages_total)
            pf_z = ph2 * p.Hkv + (u2 % p.Hkv);
        }
        if (pf_z >= 0) {
#pragma unroll
          for (int hh = 0; hh < L::kHalves; ++hh) {
            tma_prefetch_3d(&tmK, hh * 64, 0, pf_z);
            tma_prefetch_3d(&tmV, hh * 64, 0, pf_z);
          }
        }
        if (lane < 4) s_stage_lp[st][lane] = (lane < ppt && my_ph >= 0) ? my_lp : -1;
        const unsigned real = __ballot_sync(0xffffffffu, my_ph >= 0);
        __syncwarp();
        if (lane == 0)
          mbar_arrive_expect_tx(BAR(B_FULL + st), (uint32_t)__popc(real) * L::kHalves * 2u * (uint32_t)p.P * 128u);
        __syncwarp();
        if (my_ph >= 0) {
          const uint32_t dK = aKV + st * 2 * L::kTileBytes, dV = dK + L::kTileBytes;
          const int z = my_ph * p.Hkv + sg.h;
#pragma unroll
          for (int hh = 0; hh < L::kHalves; ++hh) {
            const uint32_t off = hh * (kStageTokens * 128) + lane * (p.P * 128);
            tma_load_3d(dK + off, &tmK, BAR(B_FULL + st), hh * 64, 0, z, pol);
            tma_load_3d(dV + off, &tmV, BAR(B_FULL + st), hh * 64, 0, z, pol);
          }
        }
      }
      x = sg.end;
    }
    // drain: wait until every issued copy has landed
    if (lane == 0)
      for (int k = max(0, g - NS); k < g; ++k) mbar_wait_drain(BAR(B_FULL + k % NS), (k / NS) & 1, p.status);
  } else if (warp == kMmaWarp) {
    // ======================================================= MMA issuer
    // QK runs two stages ahead of PV: after PV(g) (softmax(g) done, so S[g&1]
    // is free) comes QK(g+2); the two softmax warpgroups then overlap.
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(M, kStageTokens, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(M, D, false, true);
      Cursor qc = cursor_begin(p, s_prefix, lo, hi, W, ppt);
      Cursor pc = qc;
      int oe_seg = 0;                                    // segments whose O buffers are known free
      bool ok = true;
      // Descriptor bases; advancing along K inside a 128-byte swizzle row is
      // a 32-byte (2-unit) step of the start address, a 64-column half of
      // Q/K is M*128 / 64*128 bytes further, a 16-token step of V is 2048 bytes.
      const uint64_t dQ0 = smem_desc_sw128(aQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(aKV, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(aKV + L::kTileBytes, kStageTokens * 128, 1024);
      const uint64_t dP0 = smem_desc_sw128(aP, 16, 1024);
      constexpr uint64_t kQBuf = L::kQBytes >> 4, kQHalf = (M * 128) >> 4;
      constexpr uint64_t kStage = (2 * L::kTileBytes) >> 4, kKHalf = (kStageTokens * 128) >> 4;
      constexpr uint64_t kPBuf = L::kPBytes >> 4, kVStep = (16 * 128) >> 4;
      auto issue_qk = [&]() -> bool {
        if (qc.j == 0 && !mbar_wait(BAR(B_QFULL + (qc.s & 1)), (qc.s >> 1) & 1, &s_abort, p.status)) return false;
        const int st = qc.g % NS;
        if (!mbar_wait(BAR(B_FULL + st), (qc.g / NS) & 1, &s_abort, p.status)) return false;
        tc_fence_after();
        const uint64_t qd = dQ0 + (uint64_t)(qc.s & 1) * kQBuf;
        const uint64_t kd = dK0 + (uint64_t)st * kStage;
        const uint32_t dS = tmem + L::kColS + (qc.g & 1) * kStageTokens;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(kk & 3) * 2;
          umma_f16(dS, qd + (kk >> 2) * kQHalf + off, kd + (kk >> 2) * kKHalf + off, idQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(BAR(B_SFULL + (qc.g & 1)));
        if (qc.j == qc.nst - 1) umma_commit(BAR(B_QEMPTY + (qc.s & 1)));
        cursor_next(p, s_prefix, hi, W, ppt, qc);
        return true;
      };
      for (int k = 0; k < 2 && qc.valid && ok; ++k) ok = issue_qk();
      while (ok && pc.valid) {
        const int k = pc.g & 1;
        if (pc.j <= 1 && pc.s > oe_seg) {                // first PV of a stream in a new segment
          if (!mbar_wait(BAR(B_OEMPTY), (pc.s - 1) & 1, &s_abort, p.status)) { ok = false; break; }
          oe_seg = pc.s;
        }
        if (!mbar_wait(BAR(B_PFULL + k), (pc.g >> 1) & 1, &s_abort, p.status)) { ok = false; break; }
        tc_fence_after();
        const int st = pc.g % NS;
        const uint64_t vd = dV0 + (uint64_t)st * kStage;
        const uint64_t pd = dP0 + (uint64_t)k * kPBuf;
        const uint32_t tO = tmem + L::kColO + k * D;
        const uint32_t acc0 = pc.j >= 2 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kStageTokens / 16; ++kk)
          umma_f16(tO, pd + (uint64_t)kk * 2, vd + (uint64_t)kk * kVStep, idPV, kk > 0 ? 1u : acc0);
        umma_commit(BAR(B_EMPTY + st));
        umma_commit(BAR(B_ODONE + k));
        if (pc.j >= pc.nst - 2) umma_commit(BAR(B_OFULL + k));   // stream k's last PV of the segment
        cursor_next(p, s_prefix, hi, W, ppt, pc);
        if (qc.valid && !issue_qk()) { ok = false; break; }
      }
      umma_commit(BAR(B_TD));
    }
  } else {
    // ======================================================= softmax warpgroups
    // Warpgroup w (warps 4w..4w+3) takes the stages g with g % 2 == w, with
    // its own S, P and O buffers and its own running (max, sum) per row; the
    // two partial states of a segment are merged by warpgroup 0 in the
    // epilogue. Epilogue view (32x32b TMEM loads): thread t of warp q reads
    // TMEM lane 32q+t = packed row `i`. Stage view: for M = 64 the 16x256b
    // loads give thread t rows ra = 16q + t/4 and rb = ra + 8, columns
    // 8k + 2(t%4) + {0,1}: every lane holds live data and a row's 64 columns
    // are spread over 4 threads (quad reductions by shuffles); for M = 128
    // each thread takes its own row's 64 columns.
    const int wg = warp >> 2;
    const int q4 = warp & 3;
    const int wtid = tid & 127;                          // thread index inside the warpgroup
    const int slot = (M == 64) ? (lane < 16 ? 16 * q4 + lane : M) : 32 * q4 + lane;
    const int i = slot;                                  // packed row (epilogue view)
    const bool row_ok = i < p.rows;
    const bool warp_busy = (M == 64 ? 16 * q4 : 32 * q4) < p.rows;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int ra = 16 * q4 + (lane >> 2), rb = ra + 8;   // M = 64 stage view
    const bool ok_a = ra < p.rows, ok_b = rb < p.rows;
    const int cq = 2 * (lane & 3);
    const uint32_t tO_mine = tmem + lane_base + L::kColO + wg * D;
    int g = 0, s = 0;
    int ofull_cnt[2] = {0, 0};
    bool ok = true;
    for (int x = lo; x < hi && ok; ++s) {
      const Seg sg = locate(p, s_prefix, x, hi, W);
      const int nst = (sg.npg + ppt - 1) / ppt;
      const int g0 = g;
      const int Lb = p.context_lens[sg.b];
      const int qpos = Lb - p.R + (row_ok ? i / p.G : 0);
      const int qpos_a = Lb - p.R + (ok_a ? ra / p.G : 0), qpos_b = Lb - p.R + (ok_b ? rb / p.G : 0);
      float m_run = -INFINITY, l_run = 0.f;            // M = 128 view (and epilogue)
      float m_a = -INFINITY, l_a = 0.f, m_b = -INFINITY, l_b = 0.f;   // M = 64 stage view
      for (int j = 0; j < nst; ++j, ++g) {
        if ((g & 1) != wg) continue;
        const int st = g % NS, sb = g & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_SFULL + sb), (g >> 1) & 1, &s_abort, p.status) &&
                                         mbar_wait(BAR(B_FULL + st), (g / NS) & 1, &s_abort, p.status))) {
          ok = false;
          break;
        }
        int lp4[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) lp4[pp] = s_stage_lp[st][pp];
        bool any_invalid = false, need_mask = false;
        for (int pp = 0; pp < ppt; ++pp) {
          if (lp4[pp] < 0) { any_invalid = true; continue; }
          const int last_pos = lp4[pp] * p.P + p.P - 1;
          if (last_pos >= Lb) any_invalid = true;
          if (last_pos > Lb - p.R) need_mask = true;
        }
        need_mask |= any_invalid;
        // position of stage column c, or -1 when the token does not exist
        auto col_pos = [&](int c) {
          const int pp = c / p.P;
          const int lpc = pp == 0 ? lp4[0] : pp == 1 ? lp4[1] : pp == 2 ? lp4[2] : lp4[3];
          const int pos = lpc * p.P + (c - pp * p.P);
          return (lpc >= 0 && pos < Lb) ? pos : -1;
        };
        bool rescale = false;
        float alpha = 1.f, alpha_a = 1.f, alpha_b = 1.f;
        uint32_t pk[kStageTokens / 2];
        if constexpr (M == 64) {
          if (warp_busy) {
            tc_fence_after();
            float sv[32];
            tmem_ld16x256b_x8(tmem + lane_base + L::kColS + sb * kStageTokens, sv);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int k = 0; k < 8; ++k) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int pos = col_pos(8 * k + cq + e);
                  if (pos < 0 || pos > qpos_a) sv[4 * k + e] = -INFINITY;
                  if (pos < 0 || pos > qpos_b) sv[4 * k + 2 + e] = -INFINITY;
                }
              }
            }
            float ma[8], mb[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              ma[k] = fmaxf(sv[4 * k], sv[4 * k + 1]);
              mb[k] = fmaxf(sv[4 * k + 2], sv[4 * k + 3]);
            }
#pragma unroll
            for (int w = 4; w > 0; w >>= 1)
#pragma unroll
              for (int k = 0; k < w; ++k) { ma[k] = fmaxf(ma[k], ma[k + w]); mb[k] = fmaxf(mb[k], mb[k + w]); }
            float mxa = fmaxf(ma[0], __shfl_xor_sync(0xffffffffu, ma[0], 1));
            float mxb = fmaxf(mb[0], __shfl_xor_sync(0xffffffffu, mb[0], 1));
            mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2)) * p.scale_log2;
            mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2)) * p.scale_log2;
            if (m_a == -INFINITY) m_a = mxa;
            else if (mxa > m_a + kRescaleTau) { alpha_a = ex2(m_a - mxa); m_a = mxa; l_a *= alpha_a; rescale = true; }
            if (m_b == -INFINITY) m_b = mxb;
            else if (mxb > m_b + kRescaleTau) { alpha_b = ex2(m_b - mxb); m_b = mxb; l_b *= alpha_b; rescale = true; }
            const float nua = (m_a == -INFINITY) ? 0.f : -m_a, nub = (m_b == -INFINITY) ? 0.f : -m_b;
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sbb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float e0 = ex2(fmaf(sv[4 * k], p.scale_log2, nua));
              const float e1 = ex2(fmaf(sv[4 * k + 1], p.scale_log2, nua));
              const float e2 = ex2(fmaf(sv[4 * k + 2], p.scale_log2, nub));
              const float e3 = ex2(fmaf(sv[4 * k + 3], p.scale_log2, nub));
              sa[k & 3] += e0 + e1;
              sbb[k & 3] += e2 + e3;
              pk[2 * k] = pack_bf16x2(e0, e1);
              pk[2 * k + 1] = pack_bf16x2(e2, e3);
            }
            l_a += (sa[0] + sa[1]) + (sa[2] + sa[3]);
            l_b += (sbb[0] + sbb[1]) + (sbb[2] + sbb[3]);
          }
        } else {
          if (warp_busy) {
            tc_fence_after();
            float sv[kStageTokens];
            tmem_ld32(tmem + lane_base + L::kColS + sb * kStageTokens, sv);
            tmem_ld32(tmem + lane_base + L::kColS + sb * kStageTokens + 32, sv + 32);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int c = 0; c < kStageTokens; ++c) {
                const int pos = col_pos(c);
                if (pos < 0 || pos > qpos) sv[c] = -INFINITY;
              }
            }
            float mm[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              mm[k] = sv[8 * k];
#pragma unroll
              for (int e = 1; e < 8; ++e) mm[k] = fmaxf(mm[k], sv[8 * k + e]);
            }
            const float mx = fmaxf(fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3])),
                                   fmaxf(fmaxf(mm[4], mm[5]), fmaxf(mm[6], mm[7]))) * p.scale_log2;
            if (row_ok) {
              if (m_run == -INFINITY) {
                m_run = mx;                                // O rows are still zero
              } else if (mx > m_run + kRescaleTau) {
                alpha = ex2(m_run - mx);
                m_run = mx;
                l_run *= alpha;
                rescale = true;
              }
            }
            const float nu = (m_run == -INFINITY) ? 0.f : -m_run;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kStageTokens; c += 2) {
              const float e0 = ex2(fmaf(sv[c], p.scale_log2, nu));
              const float e1 = ex2(fmaf(sv[c + 1], p.scale_log2, nu));
              ls[(c >> 1) & 3] += e0 + e1;
              pk[c / 2] = pack_bf16x2(e0, e1);
            }
            if (row_ok) l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
          }
        }
        // P[sb] and O[sb] were last used by this stream's PV(g-2)
        if (g >= 2 && !__all_sync(0xffffffffu, mbar_wait(BAR(B_ODONE + sb), ((g - 2) >> 1) & 1, &s_abort, p.status))) {
          ok = false;
          break;
        }
        if (warp_busy) {
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            if constexpr (M == 64) {
#pragma unroll
              for (int c0 = 0; c0 < D; c0 += 64) {
                float o[32];
                tmem_ld16x256b_x8(tO_mine + c0, o);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  o[4 * k] *= alpha_a; o[4 * k + 1] *= alpha_a;
                  o[4 * k + 2] *= alpha_b; o[4 * k + 3] *= alpha_b;
                }
                tmem_st16x256b_x8(tO_mine + c0, o);
              }
            } else {
              for (int c0 = 0; c0 < D; c0 += 32) {
                float o[32];
                tmem_ld32(tO_mine + c0, o);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] *= alpha;
                tmem_st32(tO_mine + c0, o);
              }
            }
            tmem_wait_st();
          }
          uint8_t* pbuf = sP + sb * L::kPBytes;
          if constexpr (M == 64) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (ok_a) *reinterpret_cast<uint32_t*>(pbuf + ra * 128 + ((k ^ (ra & 7)) << 4) + 2 * cq) = pk[2 * k];
              if (ok_b) *reinterpret_cast<uint32_t*>(pbuf + rb * 128 + ((k ^ (rb & 7)) << 4) + 2 * cq) = pk[2 * k + 1];
            }
          } else if (row_ok) {
            uint8_t* prow = pbuf + slot * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(prow + ((c ^ (slot & 7)) << 4)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
        if (any_invalid) {
          // zero the V rows of tokens that do not exist (beyond L, missing
          // pages) so that 0 * garbage cannot reach O
          uint8_t* sV = sKV + st * 2 * L::kTileBytes + L::kTileBytes;
          for (int idx = wtid; idx < kStageTokens * L::kHalves * 8; idx += 128) {
            const int t = idx / (L::kHalves * 8);
            const int rem = idx - t * (L::kHalves * 8);
            if (col_pos(t) < 0)
              *reinterpret_cast<uint4*>(sV + (rem >> 3) * (kStageTokens * 128) + t * 128 + (rem & 7) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PFULL + sb));
      }
      if (!ok) break;
      if constexpr (M == 64) {
        // stage view -> epilogue view: total l over the quad, then row 16q + t
        // (t < 16) takes its values from quad 4(t % 8), row a for t < 8, b above
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        const int src = 4 * (lane & 7);
        const float la = __shfl_sync(0xffffffffu, l_a, src), lb = __shfl_sync(0xffffffffu, l_b, src);
        const float mva = __shfl_sync(0xffffffffu, m_a, src), mvb = __shfl_sync(0xffffffffu, m_b, src);
        l_run = (lane & 8) ? lb : la;
        m_run = (lane & 8) ? mvb : mva;
      }
      // ---- segment epilogue: warpgroup 1 hands its (max, sum) to warpgroup 0
      const bool has0 = nst >= 2 || (g0 & 1) == 0, has1 = nst >= 2 || (g0 & 1) == 1;
      if (wg == 1 && row_ok) {
        s_ml[s & 1][0][i] = m_run;
        s_ml[s & 1][1][i] = l_run;
      }
      asm volatile("bar.sync 2, 256;" ::: "memory");
      if (wg == 1) { x = sg.end; continue; }
      bool w = true;
      if (has0) w = mbar_wait(BAR(B_OFULL + 0), ofull_cnt[0] & 1, &s_abort, p.status);
      if (w && has1) w = mbar_wait(BAR(B_OFULL + 1), ofull_cnt[1] & 1, &s_abort, p.status);
      ofull_cnt[0] += has0;
      ofull_cnt[1] += has1;
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float m0 = has0 ? m_run : -INFINITY, l0 = has0 ? l_run : 0.f;
      float m1 = -INFINITY, l1 = 0.f;
      if (has1 && row_ok) { m1 = s_ml[s & 1][0][i]; l1 = s_ml[s & 1][1][i]; }
      const float mm = fmaxf(m0, m1);
      const float w0 = (m0 == -INFINITY || l0 == 0.f) ? 0.f : ex2(m0 - mm);
      const float w1 = (m1 == -INFINITY || l1 == 0.f) ? 0.f : ex2(m1 - mm);
      const float lt = l0 * w0 + l1 * w1;
      const bool single = sg.nseg == 1;
      const int slot_idx = sg.unit + blockIdx.x;           // partial slot of (unit, this CTA)
      const size_t pi = (size_t)slot_idx * p.rows + (row_ok ? i : 0);
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
      if (warp_busy) {
        const uint32_t tO0 = tmem + lane_base + L::kColO, tO1 = tO0 + D;
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32], o1[32];
          if (has0) { tmem_ld32(tO0 + c0, o); } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = 0.f;
          }
          if (has1) tmem_ld32(tO1 + c0, o1);
          tmem_wait_ld();
          if (!row_ok) continue;
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = o[c] * w0 + (has1 ? o1[c] * w1 : 0.f);
          if (single) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + out_row_offset(p, sg.b, sg.h, i) * D + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 8)
              *reinterpret_cast<uint4*>(dst + c) = make_uint4(
                  pack_bf16x2(o[c] * inv_l, o[c + 1] * inv_l), pack_bf16x2(o[c + 2] * inv_l, o[c + 3] * inv_l),
                  pack_bf16x2(o[c + 4] * inv_l, o[c + 5] * inv_l), pack_bf16x2(o[c + 6] * inv_l, o[c + 7] * inv_l));
          } else {
            float* dst = p.part_o + pi * D + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(B_OEMPTY));
      if (row_ok) {
        if (single) {
          if (p.lse) p.lse[out_row_offset(p, sg.b, sg.h, i)] = lt > 0.f ? (mm + log2f(lt)) * kLn2 : -INFINITY;
        } else {
          p.part_ml[pi * 2] = lt > 0.f ? mm : -INFINITY;
          p.part_ml[pi * 2 + 1] = lt;
        }
      }
      if (!single) {
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (wtid == 0) s_ticket = atomicAdd(p.tickets + sg.unit, 1u);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (s_ticket == sg.nseg - 1) {
          __threadfence();
          combine_partials<__nv_bfloat16>(p, sg.b, sg.h, sg.first_cta + sg.unit, sg.nseg, 128);
          if (wtid == 0) p.tickets[sg.unit] = 0u;
        }
      }
      x = sg.end;
    }
  }

  // ---- teardown: every role is done; wait for the MMAs, free TMEM
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    if (lane == 0) mbar_wait_drain(BAR(B_TD), 0, p.status);
    __syncwarp();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int M, int D>
cudaError_t launch_tc(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  CUtensorMap mk, mv;
  if (!make_cache_map(&mk, kv.k_cache, kv) || !make_cache_map(&mv, kv.v_cache, kv)) {
    *api = S3R_ERR_CUDA;
    return cudaErrorInvalidValue;
  }
  const size_t smem = Lay<M, D>::kDynBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<M, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = device_sm_count();
  if (grid > kMaxPersistentCtas) grid = kMaxPersistentCtas;
  return launch_kernel(attn_tc_kernel<M, D>, dim3(grid), dim3(kThreads), smem, st, 1, mk, mv, p);
}

}  // namespace

cudaError_t launch_attention_tc(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  *api = S3R_OK;
  const bool small = p.rows <= 64;
  if (kv.head_dim == 64) return small ? launch_tc<64, 64>(kv, p, st, api) : launch_tc<128, 64>(kv, p, st, api);
  return small ? launch_tc<64, 128>(kv, p, st, api) : launch_tc<128, 128>(kv, p, st, api);
}

}  // namespace s3r
