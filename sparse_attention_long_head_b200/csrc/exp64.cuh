// fp64 exponential of non-positive arguments, shared by the block-score
// kernel (FlashPrefill-style discovery) and the threshold select.
#pragma once
#include <cstdint>

namespace vs {

// e^x for x <= 0, branch-free, after Tang's table-driven method (P. T. P.
// Tang, "Table-driven implementation of the exponential function in IEEE
// floating-point arithmetic", ACM TOMS 15(2), 1989): x = (32 k + j) ln2/32 +
// r with |r| <= ln2/64 (r from a two-constant reduction; n ln2/32 of the
// high constant is exact for |n| < 2^17), e^r by its degree-5 Taylor
// polynomial (truncation below 2e-15 relative), times tab[j] = 2^(j/32),
// times 2^k by an exponent add.  n = round(32 x / ln2) comes from adding
// 1.5 * 2^52 in the same fma (the sum's low mantissa bits are then n, in
// two's complement, and subtracting the constant back is exact), so no
// float-integer conversion -- slow on this GPU -- is needed.  Arguments
// below -700 (e^-700 < 1e-304, negligible against the sums of at least 1
// it feeds) and -inf give 0.
constexpr double kExpInvStep = 46.16624130844683;       // 32 / ln 2
constexpr double kExpStepHi = 0.021660849392446835;     // ln 2 / 32, 36 significant bits
constexpr double kExpStepLo = 5.145609244655338e-14;    // ln 2 / 32 - kExpStepHi
constexpr double kExpShifter = 6755399441055744.0;      // 1.5 * 2^52
__device__ __forceinline__ double exp_nonpos(double x, const double* tab) {
  const double xc = fmax(x, -700.0);
  const double sh = fma(xc, kExpInvStep, kExpShifter);
  const int n = __double2loint(sh);
  const double nd = sh - kExpShifter;
  const double r = fma(nd, -kExpStepLo, fma(nd, -kExpStepHi, xc));
  double p = fma(r, 1.0 / 120.0, 1.0 / 24.0);
  p = fma(r, p, 1.0 / 6.0);
  p = fma(r, p, 0.5);
  p = fma(r, p, 1.0);
  p = fma(r, p, 1.0);
  const double v = tab[n & 31] * p;  // in [2^-1/64, 2^(31/32 + 1/64)): exponent field 1022..1023
  const double e = __hiloint2double(__double2hiint(v) + ((n >> 5) << 20), __double2loint(v));
  return x >= -700.0 ? e : 0.0;
}

__device__ __forceinline__ void exp_table_init(double* tab) {
  for (int j = threadIdx.x; j < 32; j += blockDim.x) tab[j] = exp2((double)j / 32.0);
}

}  // namespace vs
