// Token-major persistent tcgen05 attention for up to 64 packed query rows
// per (sequence, KV head): the S3R sparse draft step (G rows) and the dense
// verify step (G x (gamma + 1) rows) ("S3R: Fast and Faithful RL Rollouts
// via Self-Sparse Speculative Decoding", weekinpapers.com, Abstract: sparse
// attention over selected pages proposes, full attention over the complete
// KV history verifies, both over one shared paged cache).
//
// Decode attention has few query rows and many keys, so the contraction is
// laid out with the keys in the MMA's M dimension: every 128-token stage of
// K/V read from HBM feeds
//   S^T = K Q^T   (M = 128 tokens, N = rows rounded up to 16, K = D)
//   O^T += V^T P^T (M = D, N, K = 128 tokens),
// both fp32 in TMEM: 16 MMA instructions per 128 tokens at D = 128, where a
// rows-major M = 64 tile needs 24 and wastes most of its rows. The softmax
// thread t owns token t of the stage (TMEM lane t of S^T) and the NR real
// rows (rounded up to 8; N, the MMA's, is a multiple of 16), so the per-row
// sums stay in registers, P^T is written one token per thread, and the row
// maximum needs a cross-thread reduction only when some score exceeds the
// row's reference by more than 2^8 (the reference is lazy: O^T columns and
// the sums always share it, so the result is exact).
//
// Work partition (stream-K): the flattened (sequence, KV head, page) list is
// split into one contiguous range per CTA (s3r_attn_sched.cuh); a unit split
// over several CTAs is merged by log-sum-exp in the epilogue of the last CTA
// to finish (atomic ticket, no waiting).
//
// Warp roles (192 threads): warps 0-3 softmax and epilogue (thread = token);
// warp 4 producer (page ids, TMA into an NS-stage ring; an L2 prefetch ahead
// of the ring measured slower); warp 5 MMA issuer and TMEM owner: it polls its
// barriers and issues whichever MMA is ready (PV(k) once P(k) is written,
// QK(k) once stage k's K has landed and PV(k - 2) is issued; K and V land on
// separate barriers, so V's transfer overlaps QK(k) and softmax(k)). Two P buffers where
// they fit, so softmax(k) waits only for PV(k - 2). The softmax warps also
// stage each segment's Q (fetched into registers one segment ahead).
#include <cuda_bf16.h>

#include <cmath>

#include "s3r_attn_common.cuh"
#include "s3r_attn_sched.cuh"
#include "s3r_device.cuh"
#include "s3r_internal.h"
#include "s3r_tok_common.cuh"

namespace s3r {
namespace {

constexpr int kTokThreads = 192;
constexpr int kTokProducer = 4;
constexpr int kTokMma = 5;

// N: packed rows of the MMA (a multiple of 16); NR <= N: rows the softmax
// handles (the real rows rounded up to 8). Columns NR..N-1 of S^T and O^T
// belong to padding rows (zero queries): their P is zero and they are never
// read back.
template <int N, int NR, int D>
__global__ void __launch_bounds__(kTokThreads, 1)
attn_tok_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const AttnParams p) {
  using L = TokLay<N, D>;
  constexpr int NS = L::kNS;
  extern __shared__ __align__(1024) uint8_t dyn_raw[];
  uint8_t* dyn = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t s_bar[3 * NS + 8];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_ticket;
  __shared__ int4 s_pend[kMaxPend];             // units this CTA combines at its end: (b, h, slot0, nseg)
  __shared__ int s_npend;
  __shared__ int s_prefix[kMaxSeqs + 1];
  __shared__ int s_stage_lp[NS][8];
  __shared__ int s_roff[64];                    // output row of packed row r relative to (b, h)
  __shared__ float s_red[4][64];
  __shared__ float s_mx[64];                    // stage maximum per row (raw score)
  __shared__ __align__(16) float s_nu[64];      // -(reference) per row, log2 units
  __shared__ __align__(16) float s_alpha[64];   // rescale factor / 1 / l per row
  __shared__ unsigned long long s_tmask[64];    // tree: ancestors-or-self of each round node
  __shared__ unsigned long long s_pmask[64];    // tree: packed rows that see each round slot

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
  if (tid < 64) s_roff[tid] = (tid / p.G) * p.Hq + (tid % p.G);
  __syncthreads();
  // Earlier kernels' results (page lists) and their use of the outputs and
  // workspace are ordered by griddepcontrol.wait, taken by each role right
  // before it needs them: the producer before the page ids, the softmax
  // warps after fetching their first Q.
  if (blockIdx.x == 0) {
    pdl_wait();
    // unusable lengths: flag them, give their rows zero output and lse -inf
    for (int b = 0; b < p.S; ++b) {
      if (!bad_context(p, p.context_lens[b])) continue;
      if (tid == 0) flag_status(p.status, S3R_DEV_BAD_CONTEXT_LEN);
      for (int h = 0; h < p.Hkv; ++h) write_empty_unit<__nv_bfloat16>(p, b, h, tid, kTokThreads);
    }
  }
  const int total = s_prefix[p.S];
  // Sparse draft: when the (sequence, KV head) units nearly fill the grid
  // (at least 4/5 of it), each CTA takes one whole unit of B pages instead of
  // an equal share: no unit is split, so no partials, tickets or merges (the
  // idle CTAs cost less than the split units on the 16 x 16K workload).
  int W = (total + gridDim.x - 1) / gridDim.x;
  if (p.page_list && W < p.budget && p.S * p.Hkv * 5 >= (int)gridDim.x * 4) W = p.budget;
  const int lo = blockIdx.x * W, hi = min(total, lo + W);
  if (lo >= hi) {                                       // uniform over the CTA
    pdl_wait();
    return;
  }
  const int ppt = kTok / p.P;                           // pages per stage

  const uint32_t bar0 = smem_addr(&s_bar[0]);
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  // PFULL[k] / ODONE[k]: completed by softmax(g) / PV(g) for g % 2 == k.
  // softmax(g + 1) need not wait for PV(g) (two P buffers), so one PFULL
  // barrier could complete two phases before the MMA thread tests the first;
  // with one barrier per parity, P(g + 2) waits for PV(g) and no barrier gets
  // two phases ahead of its waiter.
  // FULL[st]: the stage's K landed (and its page ids written); FULLV[st]: its V
  const int B_FULL = 0, B_EMPTY = NS, B_SFULL = 2 * NS, B_PFULL = 2 * NS + 2, B_ODONE = 2 * NS + 4,
            B_QFULL = 2 * NS + 6, B_TD = 2 * NS + 7, B_FULLV = 2 * NS + 8;
  constexpr int PB = L::kPBufs;
  uint8_t* sQ = dyn;
  uint8_t* sP = dyn + L::kOffP;
  uint8_t* sKV = dyn + L::kOffKV;
  const uint32_t aQ = smem_addr(sQ), aP = smem_addr(sP), aKV = smem_addr(sKV);

  if (warp == kTokMma) {
    tmem_alloc(smem_addr(&s_tmem), 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(BAR(B_FULL + i), 1);
      mbar_init(BAR(B_FULLV + i), 1);
      mbar_init(BAR(B_EMPTY + i), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SFULL + 1), 1);
    mbar_init(BAR(B_PFULL), 128);
    mbar_init(BAR(B_PFULL + 1), 128);
    mbar_init(BAR(B_ODONE), 1);
    mbar_init(BAR(B_ODONE + 1), 1);
    mbar_init(BAR(B_QFULL), 128);
    mbar_init(BAR(B_TD), 1);
    s_abort = 0;
    s_npend = 0;
    fence_barrier_init();
  }
  if (warp == kTokProducer && lane == 0) { prefetch_tensormap(&tmK); prefetch_tensormap(&tmV); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == kTokProducer) {
    // ======================================================= producer warp
    // A page list is an earlier kernel's output (wait for it first); the
    // block table and the K/V cache are inputs, so the dense path resolves
    // its first page ids and issues its first NS ring stages before the wait.
    if (p.page_list) pdl_wait();
    const uint64_t pol = l2_policy_evict_first();
    // page-id windows of 32 flattened positions: lane k of a window holds
    // position wbase + k. w0 = in use, w1 = phys loads in flight, w2 = lp
    // loads in flight (with the selector's physical ids, w2_pp).
    int w0_lp, w0_ph, w0_u, w1_lp, w1_ph, w1_u, w2_lp, w2_u, w2_pp, pp;
    auto phys_load = [&](int lp, int u, int ph_sel) {
      if (lp < 0) return -1;
      if (p.page_phys) return ph_sel;
      const int b = u / p.Hkv;
      const int n_b = (p.context_lens[b] + p.P - 1) / p.P;
      if (lp >= n_b) { flag_status(p.status, S3R_DEV_BAD_PAGE_ID); return -1; }
      return p.block_table[(size_t)b * p.max_pages + lp];
    };
    int wbase = lo;
    page_of(p, s_prefix, wbase + lane, hi, W, &w0_lp, &w0_u, &pp);
    w0_ph = phys_load(w0_lp, w0_u, pp);
    page_of(p, s_prefix, wbase + 32 + lane, hi, W, &w1_lp, &w1_u, &pp);
    w1_ph = phys_load(w1_lp, w1_u, pp);
    page_of(p, s_prefix, wbase + 64 + lane, hi, W, &w2_lp, &w2_u, &w2_pp);
    bool waited = p.page_list != nullptr;
    int g = 0;
    bool ok = true;
    for (int x = lo; x < hi && ok;) {
      const Seg sg = locate(p, s_prefix, x, hi, W);
      const int nst = (sg.npg + ppt - 1) / ppt;
      for (int j = 0; j < nst; ++j, ++g) {
        const int st = g % NS;
        if (g == NS && !waited) {                        // the ring's first fill went out before it
          pdl_wait();
          waited = true;
        }
        // the stage's page ids first (they do not need the slot), then the slot
        int my_lp = -1, my_ph = -1;
        for (int pp = 0; pp < ppt; ++pp) {
          // positions past the segment belong to the next one: the windows
          // must not move past its first page (warp-uniform)
          if (j * ppt + pp >= sg.npg) break;
          const int xp = x + j * ppt + pp;
          while (xp >= wbase + 32) {                   // advance the windows (warp-uniform)
            wbase += 32;
            w0_lp = w1_lp; w0_ph = w1_ph; w0_u = w1_u;
            w1_lp = w2_lp; w1_u = w2_u;
            w1_ph = phys_load(w1_lp, w1_u, w2_pp);
            page_of(p, s_prefix, wbase + 64 + lane, hi, W, &w2_lp, &w2_u, &w2_pp);
          }
          const int src = xp - wbase;
          const int lp = __shfl_sync(0xffffffffu, w0_lp, src & 31);
          int ph = __shfl_sync(0xffffffffu, w0_ph, src & 31);
          if (lp >= 0 && (ph < 0 || ph >= p.num_pages_total)) {
            if (lane == 0) flag_status(p.status, S3R_DEV_BAD_PAGE_ID);
            ph = -1;
          }
          if (lane == pp) { my_lp = lp; my_ph = ph; }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_EMPTY + st), ((g / NS) & 1) ^ 1, &s_abort, p.status))) {
          ok = false;
          break;
        }
        if (lane < 8) s_stage_lp[st][lane] = (lane < ppt && my_ph >= 0) ? my_lp : -1;
        const unsigned real = __ballot_sync(0xffffffffu, my_ph >= 0);
        __syncwarp();
        if (lane == 0) {
          // K and V land on separate barriers: QK(g) needs only K, so V's
          // transfer is no longer between the stage's arrival and its QK
          const uint32_t half = (uint32_t)__popc(real) * L::kHalves * (uint32_t)p.P * 128u;
          mbar_arrive_expect_tx(BAR(B_FULL + st), half);
          mbar_arrive_expect_tx(BAR(B_FULLV + st), half);
        }
        __syncwarp();
        if (my_ph >= 0) {
          const uint32_t dK = aKV + st * 2 * L::kTileBytes, dV = dK + L::kTileBytes;
          const int z = my_ph * p.Hkv + sg.h;
#pragma unroll
          for (int hh = 0; hh < L::kHalves; ++hh)
            tma_load_3d(dK + hh * (kTok * 128) + lane * (p.P * 128), &tmK, BAR(B_FULL + st), hh * 64, 0, z, pol);
#pragma unroll
          for (int hh = 0; hh < L::kHalves; ++hh)
            tma_load_3d(dV + hh * (kTok * 128) + lane * (p.P * 128), &tmV, BAR(B_FULLV + st), hh * 64, 0, z, pol);
        }
      }
      x = sg.end;
    }
    if (!waited) pdl_wait();
    // drain: wait until every issued copy has landed
    if (lane == 0)
      for (int k = max(0, g - NS); k < g; ++k) {
        mbar_wait_drain(BAR(B_FULL + k % NS), (k / NS) & 1, p.status);
        mbar_wait_drain(BAR(B_FULLV + k % NS), (k / NS) & 1, p.status);
      }
  } else if (warp == kTokMma) {
    // ======================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(kTok, N, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(D, N, true, false);
      Cursor qc = cursor_begin(p, s_prefix, lo, hi, W, ppt);
      Cursor pc = qc;
      bool ok = true;
      // K (A of S^T) and Q (B): K-major, 128-byte rows, 8-row groups 1024 B
      // apart; a K16 step is 32 bytes inside the swizzle row, the next 64
      // columns are one half-tile further. V^T (A of O^T) is M-major: the
      // two 64-dim halves one 128-token half-tile apart, 16 tokens = 2048 B.
      // P^T (B of O^T): K-major, 64-token halves N * 128 bytes apart.
      const uint64_t dQ0 = smem_desc_sw128(aQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(aKV, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(aKV + L::kTileBytes, kTok * 128, 1024);
      const uint64_t dP0 = smem_desc_sw128(aP, 16, 1024);
      constexpr uint64_t kQHalf = (N * 128) >> 4, kPHalf = (N * 128) >> 4;
      constexpr uint64_t kStage = (2 * L::kTileBytes) >> 4, kKHalf = (kTok * 128) >> 4, kVStep = (16 * 128) >> 4;
      // QK(k) needs its stage's data (first in a segment, also the segment's
      // Q) and PV(k - 2) issued (softmax(k - 2) has read S buffer k & 1);
      // PV(k) needs P(k). Each is issued as soon as it is ready, so a PV never
      // waits for a later stage's data. Bounded: no progress for the wait
      // limit flags a timeout and stops.
      auto issue_qk = [&]() {
        tc_fence_after();
        const int st = qc.g % NS;
        const uint64_t kd = dK0 + (uint64_t)st * kStage;
        const uint32_t dS = tmem + L::kColS + (qc.g & 1) * N;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(kk & 3) * 2;
          umma_f16(dS, kd + (kk >> 2) * kKHalf + off, dQ0 + (kk >> 2) * kQHalf + off, idQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(BAR(B_SFULL + (qc.g & 1)));
        cursor_next(p, s_prefix, hi, W, ppt, qc);
      };
      auto issue_pv = [&]() {
        tc_fence_after();
        const int st = pc.g % NS;
        const uint64_t vd = dV0 + (uint64_t)st * kStage;
        const uint32_t tO = tmem + L::kColO;
        const uint32_t acc0 = pc.j > 0 ? 1u : 0u;
        const uint64_t pd = dP0 + (uint64_t)(pc.g % PB) * (L::kPBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk)
          umma_f16(tO, vd + (uint64_t)kk * kVStep, pd + (kk >> 2) * kPHalf + (uint64_t)(kk & 3) * 2, idPV,
                   kk > 0 ? 1u : acc0);
        umma_commit(BAR(B_EMPTY + st));
        umma_commit(BAR(B_ODONE + (pc.g & 1)));
        cursor_next(p, s_prefix, hi, W, ppt, pc);
      };
      unsigned long long idle_since = 0;
      uint32_t spins = 0;
      while (pc.valid) {
        bool progress = false;
        if (mbar_test_wait(BAR(B_PFULL + (pc.g & 1)), (pc.g >> 1) & 1) &&
            mbar_test_wait(BAR(B_FULLV + pc.g % NS), (pc.g / NS) & 1)) {
          issue_pv();
          progress = true;
        }
        if (qc.valid && qc.g <= pc.g + 1 && (qc.j != 0 || mbar_test_wait(BAR(B_QFULL), qc.s & 1)) &&
            mbar_test_wait(BAR(B_FULL + qc.g % NS), (qc.g / NS) & 1)) {
          issue_qk();
          progress = true;
        }
        if (progress) {
          idle_since = 0;
          continue;
        }
        if ((++spins & 63u) == 0) {
          if (s_abort) { ok = false; break; }
          const unsigned long long now = globaltimer_ns();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            s_abort = 1;
            flag_status(p.status, S3R_DEV_WAIT_TIMEOUT);
            ok = false;
            break;
          }
        }
      }
      (void)ok;
      umma_commit(BAR(B_TD));
    }
  } else {
    // ======================================================= softmax warps
    // Thread t: token t of each stage (TMEM lane t of S^T), and TMEM lane t
    // of O^T in the epilogue (dimension t for D = 128; for D = 64 the M = 64
    // accumulator puts dimension 16q + l in lane 32q + l, l < 16).
    const int q4 = warp;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int d_mine = (D == 128) ? tid : (lane < 16 ? 16 * q4 + lane : -1);
    const int log2P = __ffs(p.P) - 1;
    const float c = p.scale_log2;
    constexpr int kQC = L::kQChunks;
    constexpr int kDc = D / 8;                          // 16-byte chunks per Q row
    uint4 qr[kQC];
    auto q_fetch = [&](const Seg& s) {
      const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
      const size_t base = (size_t)(s.b * p.R) * p.Hq + (size_t)s.h * p.G;
#pragma unroll
      for (int k = 0; k < kQC; ++k) {
        const int ch = tid + 128 * k, r = ch / kDc, c16 = ch - (ch / kDc) * kDc;
        qr[k] = r < p.rows ? __ldg(reinterpret_cast<const uint4*>(q + (base + s_roff[r]) * D + c16 * 8))
                           : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto q_store = [&]() {
#pragma unroll
      for (int k = 0; k < kQC; ++k) {
        const int ch = tid + 128 * k, r = ch / kDc, c16 = ch - (ch / kDc) * kDc;
        *reinterpret_cast<uint4*>(sQ + (c16 >> 3) * (N * 128) + r * 128 + (((c16 & 7) ^ (r & 7)) << 4)) = qr[k];
      }
      fence_proxy_async_smem();
      mbar_arrive(BAR(B_QFULL));
    };
    Seg sg = locate(p, s_prefix, lo, hi, W);
    q_fetch(sg);                                        // an input: no earlier kernel writes it
    pdl_wait();
    q_store();
    if constexpr (NR < N) {
      // P rows NR..N-1 (padding) are zero in both buffers for the whole run;
      // the first stage's proxy fence publishes these writes with its P
      const int half = tid >> 6, tt = tid & 63, ck = tt >> 3;
#pragma unroll
      for (int b2 = 0; b2 < PB; ++b2) {
        uint8_t* pb = sP + b2 * L::kPBytes + half * (N * 128) + (tt & 7) * 2;
#pragma unroll
        for (int r = NR; r < N; ++r)
          *reinterpret_cast<__nv_bfloat16*>(pb + r * 128 + ((ck ^ (r & 7)) << 4)) = __float2bfloat16_rn(0.f);
      }
    }
    int g = 0;
    bool ok = true;
    for (int x = lo; x < hi;) {
      const bool has_next = sg.end < hi;
      Seg nx = sg;
      if (has_next) {
        nx = locate(p, s_prefix, sg.end, hi, W);
        q_fetch(nx);                                   // lands while this segment runs
      }
      const int nst = (sg.npg + ppt - 1) / ppt;
      const int Lb = p.context_lens[sg.b];
      if (tid < N) s_nu[tid] = kNuInit;
      if (p.tree_parent) {
        // the round's nodes: ancestors-or-self of each (parents precede their
        // children; a bad entry ends the walk and is flagged), then for each
        // round slot the packed rows allowed to see it
        if (tid < p.R) {
          const int32_t* par = p.tree_parent + (size_t)sg.b * p.R;
          unsigned long long m = 1ull << tid;
          int v = tid;
          for (int guard = 0; guard < 64 && v > 0; ++guard) {
            const int pv = par[v];
            if (pv < 0 || pv >= v) { flag_status(p.status, S3R_DEV_BAD_TREE); break; }
            m |= 1ull << pv;
            v = pv;
          }
          if (tid == 0 && par[0] != -1) flag_status(p.status, S3R_DEV_BAD_TREE);
          s_tmask[tid] = m;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (tid < p.R) {
          unsigned long long pm = 0;
          for (int r = 0; r < p.rows; ++r)
            if ((s_tmask[r / p.G] >> tid) & 1ull) pm |= 1ull << r;
          s_pmask[tid] = pm;
        }
      }
      float l[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) l[r] = 0.f;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      bool abort_all = false;
      for (int j = 0; j < nst; ++j, ++g) {
        const int st = g % NS, sb = g & 1;
        ok &= mbar_wait(BAR(B_SFULL + sb), (g >> 1) & 1, &s_abort, p.status) &&
              mbar_wait(BAR(B_FULL + st), (g / NS) & 1, &s_abort, p.status);
        tc_fence_after();
        // this thread's token: position, existence, causal mask of the rows
        const int lp = s_stage_lp[st][tid >> log2P];
        const int pos = lp * p.P + (tid & (p.P - 1));
        const bool valid = lp >= 0 && pos < Lb;
        const int excess = pos - (Lb - p.R);
        // packed rows that may not see this token: a token that does not exist
        // hides from all; inside the round, the causal chain hides from the
        // rows of earlier positions, a tree from the rows of non-descendants
        unsigned long long hide = 0;
        if (!valid) hide = ~0ull;
        else if (p.tree_parent) hide = excess >= 0 ? ~s_pmask[excess] : 0ull;
        else if (excess > 0) {
          const int nm = min(N, p.G * excess);
          hide = nm >= 64 ? ~0ull : ((1ull << nm) - 1ull);
        }
        float s[NR];
        auto load_s = [&]() {
          tmem_ld_cols<NR>(tmem + lane_base + L::kColS + sb * N, s);
          tmem_wait_ld();
          if (hide) {
#pragma unroll
            for (int r = 0; r < NR; ++r)
              if ((hide >> r) & 1ull) s[r] = -INFINITY;
          }
        };
        load_s();
        float ymax = -INFINITY;
#pragma unroll
        for (int r = 0; r < NR; r += 4) {
          const float4 v = *reinterpret_cast<const float4*>(&s_nu[r]);
          ymax = fmaxf(fmaxf(ymax, fmaf(s[r], c, v.x)), fmaf(s[r + 1], c, v.y));
          ymax = fmaxf(fmaxf(ymax, fmaf(s[r + 2], c, v.z)), fmaf(s[r + 3], c, v.w));
        }
        // one barrier per stage: stop together, or raise the references together
        const int cnt = wg_count(!ok || ymax > kTau);
        bool rescale_o = false;
        if (cnt > 0) {
          if (wg_count(!ok) > 0) { abort_all = true; break; }
          // stage maximum per row (S^T is intact until PFULL), then reload
          wg_rows_reduce<NR, true>(s, s_red, s_mx, q4, lane, tid);
          if (tid < NR) {
            const float m_old = -s_nu[tid];
            const float m_new = fmaxf(m_old, s_mx[tid] * c);
            s_alpha[tid] = ex2(m_old - m_new);
            s_nu[tid] = -m_new;
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
          for (int r = 0; r < NR; r += 4) {
            const float4 a = *reinterpret_cast<const float4*>(&s_alpha[r]);
            l[r] *= a.x; l[r + 1] *= a.y; l[r + 2] *= a.z; l[r + 3] *= a.w;
          }
          load_s();
          rescale_o = j > 0;
        }
        // s <- P = 2^(s c - m_ref), row sums
#pragma unroll
        for (int r = 0; r < NR; r += 4) {
          const float4 v = *reinterpret_cast<const float4*>(&s_nu[r]);
          s[r] = ex2(fmaf(s[r], c, v.x));
          s[r + 1] = ex2(fmaf(s[r + 1], c, v.y));
          s[r + 2] = ex2(fmaf(s[r + 2], c, v.z));
          s[r + 3] = ex2(fmaf(s[r + 3], c, v.w));
          l[r] += s[r]; l[r + 1] += s[r + 1]; l[r + 2] += s[r + 2]; l[r + 3] += s[r + 3];
        }
        // P buffer g % PB was last read by PV(g - PB); a rescale of O^T also
        // needs PV(g - 1) done
        const int gw = g - ((rescale_o || PB == 1) ? 1 : 2);
        if (gw >= 0) ok &= mbar_wait(BAR(B_ODONE + (gw & 1)), (gw >> 1) & 1, &s_abort, p.status);
        tc_fence_after();
        if (rescale_o) {
          float o[NR];
          tmem_ld_cols<NR>(tmem + lane_base + L::kColO, o);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < NR; ++r) o[r] *= s_alpha[r];
          tmem_st_cols<NR>(tmem + lane_base + L::kColO, o);
          tmem_wait_st();
        }
        {
          const int half = tid >> 6, tt = tid & 63;
          uint8_t* pb = sP + (g % PB) * L::kPBytes + half * (N * 128) + (tt & 7) * 2;
          const int ck = tt >> 3;
#pragma unroll
          for (int r = 0; r < NR; ++r)
            *reinterpret_cast<__nv_bfloat16*>(pb + r * 128 + ((ck ^ (r & 7)) << 4)) = __float2bfloat16_rn(s[r]);
        }
        if (!valid) {
          // a token that does not exist (beyond L, or a missing page): zero
          // its V row so that 0 * stale data cannot reach O (once the
          // stage's V has landed, so that the copy cannot overwrite it)
          ok &= mbar_wait(BAR(B_FULLV + st), (g / NS) & 1, &s_abort, p.status);
          uint8_t* sV = sKV + st * 2 * L::kTileBytes + L::kTileBytes + tid * 128;
#pragma unroll
          for (int hh = 0; hh < L::kHalves; ++hh)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              *reinterpret_cast<uint4*>(sV + hh * (kTok * 128) + k * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PFULL + (g & 1)));
      }
      if (abort_all) break;
      // ---- the last QK of this segment is done: stage the next segment's Q
      if (has_next) q_store();
      // ---- segment epilogue: row sums, then O^T / l
      wg_rows_reduce<NR, false>(l, s_red, s_alpha, q4, lane, tid);
      const bool single = sg.nseg == 1;
      const int slot_idx = sg.unit + blockIdx.x;          // partial slot of (unit, this CTA)
      const size_t rowbase = (size_t)(sg.b * p.R) * p.Hq + (size_t)sg.h * p.G;
      if (tid < p.rows) {
        const float lt = s_alpha[tid], m = -s_nu[tid];
        if (single) {
          if (p.lse) p.lse[rowbase + s_roff[tid]] = lt > 0.f ? (m + log2f(lt)) * kLn2 : -INFINITY;
        } else {
          const size_t pi = (size_t)slot_idx * p.rows + tid;
          p.part_ml[pi * 2] = lt > 0.f ? m : -INFINITY;
          p.part_ml[pi * 2 + 1] = lt;
        }
        s_alpha[tid] = lt > 0.f ? 1.f / lt : 0.f;
      }
      ok &= mbar_wait(BAR(B_ODONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, &s_abort, p.status);   // PV of the last stage
      tc_fence_after();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      {
        float o[NR];
        tmem_ld_cols<NR>(tmem + lane_base + L::kColO, o);
        tmem_wait_ld();
        if (d_mine >= 0) {
          if (single) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + rowbase * D + d_mine;
#pragma unroll
            for (int r = 0; r < NR; ++r)
              if (r < p.rows) dst[(size_t)s_roff[r] * D] = __float2bfloat16_rn(o[r] * s_alpha[r]);
          } else {
            float* dst = p.part_o + (size_t)slot_idx * p.rows * D + d_mine;
#pragma unroll
            for (int r = 0; r < NR; ++r)
              if (r < p.rows) dst[(size_t)r * D] = o[r];
          }
        }
      }
      tc_fence_before();
      if (!single) {
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (tid == 0) s_ticket = atomicAdd(p.tickets + sg.unit, 1u);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (s_ticket == sg.nseg - 1) {
          // this CTA finished the unit last: merge its partials after the
          // CTA's own streaming is done (immediately if the list is full)
          if (s_npend < kMaxPend) {
            if (tid == 0) s_pend[s_npend] = make_int4(sg.b, sg.h, sg.first_cta + sg.unit, sg.nseg);
          } else {
            __threadfence();
            combine_partials<__nv_bfloat16>(p, sg.b, sg.h, sg.first_cta + sg.unit, sg.nseg, 128);
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (tid == 0) {
            if (s_npend < kMaxPend) ++s_npend;
            p.tickets[sg.unit] = 0u;
          }
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");    // s_alpha / s_nu reads done
      x = sg.end;
      sg = nx;
    }
    // ---- deferred combines of the units this CTA finished last (skipped,
    // together, after a failed wait)
    if (wg_count(!ok) == 0) {
      __threadfence();
      for (int k = 0; k < s_npend; ++k) {
        const int4 u = s_pend[k];
        combine_partials<__nv_bfloat16>(p, u.x, u.y, u.z, u.w, 128);
      }
    }
  }

  // ---- teardown: every role is done; wait for the MMAs, free TMEM
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kTokMma) {
    tc_fence_after();
    if (lane == 0) mbar_wait_drain(BAR(B_TD), 0, p.status);
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

template <int N, int NR, int D>
cudaError_t launch_tok(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  CUtensorMap mk, mv;
  if (!make_cache_map(&mk, kv.k_cache, kv) || !make_cache_map(&mv, kv.v_cache, kv)) {
    *api = S3R_ERR_CUDA;
    return cudaErrorInvalidValue;
  }
  const size_t smem = TokLay<N, D>::kDynBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tok_kernel<N, NR, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = device_sm_count();
  if (grid > kMaxPersistentCtas) grid = kMaxPersistentCtas;
  return launch_kernel(attn_tok_kernel<N, NR, D>, dim3(grid), dim3(kTokThreads), smem, st, 1, mk, mv, p);
}

// MMA rows N: the packed rows rounded up to 16; softmax rows NR: to 8 for
// N = 16 and 32 (the draft's G rows, verify's G (gamma + 1) rows of the
// workloads), N itself for 48 and 64.
template <int D>
cudaError_t launch_tok_rows(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  const bool half = (p.rows & 15) != 0 && (p.rows & 15) <= 8;
  if (p.rows <= 16) return half ? launch_tok<16, 8, D>(kv, p, st, api) : launch_tok<16, 16, D>(kv, p, st, api);
  if (p.rows <= 32) return half ? launch_tok<32, 24, D>(kv, p, st, api) : launch_tok<32, 32, D>(kv, p, st, api);
  if (p.rows <= 48) return launch_tok<48, 48, D>(kv, p, st, api);
  return launch_tok<64, 64, D>(kv, p, st, api);
}

}  // namespace

cudaError_t launch_attention_tok(const s3r_paged_kv& kv, const AttnParams& p, cudaStream_t st, s3r_status* api) {
  *api = S3R_OK;
  return kv.head_dim == 64 ? launch_tok_rows<64>(kv, p, st, api) : launch_tok_rows<128>(kv, p, st, api);
}

}  // namespace s3r
