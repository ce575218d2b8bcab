// Work partition shared by the persistent tensor-core attention kernels.
//
// The work of one call is the flattened list of (sequence, KV head, page)
// triples: all n_b pages of every KV head (verify) or the min(B, n_b)
// selected pages (draft), sequences in order, KV heads in order. s_prefix[b]
// (kept in shared memory) is the flattened position of sequence b's first
// page. CTA c takes positions [c*W, (c+1)*W); each maximal piece of one
// (sequence, KV head) unit inside that range is a segment.
#pragma once

#include "s3r_attn_common.cuh"

namespace s3r {

// One maximal piece of a (sequence, KV head) unit inside a CTA's range.
struct Seg {
  int b, h;        // sequence, KV head
  int k0, npg;     // first page-list index and number of pages
  int end;         // flattened position after the segment
  int unit;        // b * Hkv + h
  int first_cta;   // first CTA whose range holds part of the unit
  int nseg;        // number of CTAs sharing the unit
};

// s_prefix[b] = sum over sequences before b of Hkv * pages(b)
__device__ __forceinline__ Seg locate(const AttnParams& p, const int* s_prefix, int x, int hi, int W) {
  int lo_b = 0, hi_b = p.S - 1;
  while (lo_b < hi_b) {                      // first b with prefix[b+1] > x
    const int mid = (lo_b + hi_b) >> 1;
    if (s_prefix[mid + 1] > x) hi_b = mid; else lo_b = mid + 1;
  }
  Seg s;
  s.b = lo_b;
  const int pages = (s_prefix[lo_b + 1] - s_prefix[lo_b]) / p.Hkv;
  const int o = x - s_prefix[lo_b];
  s.h = o / pages;
  s.k0 = o - s.h * pages;
  const int ustart = s_prefix[lo_b] + s.h * pages, uend = ustart + pages;
  s.end = min(hi, uend);
  s.npg = s.end - x;
  s.unit = s.b * p.Hkv + s.h;
  s.first_cta = ustart / W;
  s.nseg = (uend - 1) / W - s.first_cta + 1;
  return s;
}

// Logical page and unit (b * Hkv + h) of flattened position x (-1 when out
// of range); with p.page_phys also the physical page id (else -1).
__device__ __forceinline__ void page_of(const AttnParams& p, const int* s_prefix, int x, int hi, int W,
                                        int* lp_out, int* u_out, int* ph_out = nullptr) {
  *lp_out = -1;
  *u_out = 0;
  if (ph_out) *ph_out = -1;
  if (x >= hi) return;
  const Seg s = locate(p, s_prefix, x, hi, W);
  *u_out = s.unit;
  const size_t i = ((size_t)s.b * p.Hkv + s.h) * p.budget + s.k0;
  *lp_out = p.page_list ? p.page_list[i] : s.k0;
  if (ph_out && p.page_phys) *ph_out = p.page_phys[i];
}

// Walk over the stages of a CTA's range, segment by segment.
struct Cursor {
  int x, s, j, nst, g;    // segment start, segment index, stage in segment, stages in segment, global stage
  bool valid;
  Seg sg;
};
__device__ __forceinline__ Cursor cursor_begin(const AttnParams& p, const int* s_prefix, int lo, int hi, int W,
                                               int ppt) {
  Cursor c;
  c.x = lo; c.s = 0; c.j = 0; c.g = 0; c.nst = 0;
  c.valid = lo < hi;
  if (c.valid) {
    c.sg = locate(p, s_prefix, lo, hi, W);
    c.nst = (c.sg.npg + ppt - 1) / ppt;
  }
  return c;
}
__device__ __forceinline__ void cursor_next(const AttnParams& p, const int* s_prefix, int hi, int W, int ppt,
                                            Cursor& c) {
  ++c.g;
  if (++c.j >= c.nst) {
    c.x = c.sg.end;
    ++c.s;
    c.j = 0;
    c.valid = c.x < hi;
    if (c.valid) {
      c.sg = locate(p, s_prefix, c.x, hi, W);
      c.nst = (c.sg.npg + ppt - 1) / ppt;
    }
  }
}


}  // namespace s3r
