// Table-driven float64 exponential shared by the sampling kernels.
#pragma once

#include <cuda_runtime.h>

namespace s3r {

// float64 exponential, table-driven (P. T. P. Tang, "Table-driven
// implementation of the exponential function in IEEE floating-point
// arithmetic", ACM Trans. Math. Software 15(2), 1989), with a 256-entry
// table: write x = (256 m + j) ln2/256 + r with |r| <= ln2/512, then
// exp(x) = 2^m * 2^(j/256) * e^r. N = 256 m + j is x * 256/ln2 rounded to an
// integer by adding 1.5 * 2^52; r = x - N ln2/256 with ln2/256 split into a
// double and its remainder (two fused multiply-adds); e^r - 1 is its Taylor
// polynomial to degree 4 (remainder < 4e-17 for |r| <= ln2/512); 2^(j/256)
// is the table `tab`. exp_tbl_core returns 2^(j/256) e^r and m.
constexpr int kExpTab = 256;
__device__ __forceinline__ double exp_tbl_core(double x, const double* tab, int* m) {
  constexpr double kInvStep = 369.32993046757463;          // 256 / ln2
  constexpr double kStepHi = 0x1.62e42fefa39efp-9;          // ln2 / 256, leading double
  constexpr double kStepLo = 0x1.abc9e3b39803fp-64;         // ln2 / 256 - kStepHi
  constexpr double kShifter = 6755399441055744.0;           // 1.5 * 2^52
  const double t = fma(x, kInvStep, kShifter);
  const int n = __double2loint(t);
  const double nd = t - kShifter;
  double r = fma(-nd, kStepHi, x);
  r = fma(-nd, kStepLo, r);
  double q = fma(r, 1.0 / 24.0, 1.0 / 6.0);
  q = fma(q, r, 0.5);
  q = fma(q, r, 1.0);
  const double tj = tab[n & (kExpTab - 1)];
  *m = n >> 8;                                              // floor(N / 256)
  return fma(tj, q * r, tj);
}
// exp(x) with 2^m put into the exponent field: within about 2 ulp for
// -707 < x < 708; outside that range the field overflows (callers fix such
// values up with exp_fixup).
__device__ __forceinline__ double exp_tbl(double x, const double* tab) {
  int m;
  const double y = exp_tbl_core(x, tab, &m);
  return __hiloint2double(__double2hiint(y) + m * (1 << 20), __double2loint(y));
}
// exp(x) given y = exp_tbl(x): outside (-707, 708) the power of two is
// applied in two exact steps (half through the exponent field, the rest as an
// exact power-of-two factor), so the result is the core value times 2^m with
// a single rounding where it is subnormal; 0 below -746, infinity above
// 709.79, NaN stays NaN. No library call, so the hot loops carry no call ABI.
__device__ __forceinline__ double exp_fixup(double x, double y, const double* tab) {
  if (x > -707.0 && x < 708.0) return y;
  if (x != x) return x;
  if (x < -746.0) return 0.0;
  if (x > 709.79) return INFINITY;
  int m;
  const double y0 = exp_tbl_core(x, tab, &m);
  const int m1 = m / 2, m2 = m - m1;                        // |m1|, |m2| <= 539: both powers are normal
  const double a = __hiloint2double(__double2hiint(y0) + m1 * (1 << 20), __double2loint(y0));
  return a * __hiloint2double((m2 + 1023) << 20, 0);
}

// 2^(j/256), j = 0..255, into shared memory (caller syncs).
__device__ __forceinline__ void fill_exp_tab(double* tab) {
  for (int j = threadIdx.x; j < kExpTab; j += blockDim.x) tab[j] = exp2(static_cast<double>(j) * (1.0 / kExpTab));
}

}  // namespace s3r
