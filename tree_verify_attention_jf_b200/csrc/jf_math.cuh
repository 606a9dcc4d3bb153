// jf_math.cuh -- float64 exp for non-positive arguments, used for the draft-logit row sums.
//
// Method: table-driven additive range reduction (P. T. P. Tang, "Table-driven implementation of the
// exponential function in IEEE floating-point arithmetic", ACM TOMS 15(2), 1989):
// x = (32 k + j) ln2 / 32 + r with integer k, j in [0, 32) and |r| <= ln2 / 64 (plus rounding), where
// ln2 / 32 is split into a 32-significant-bit head (so n * head is exact) and a tail.  Then
// e^x = 2^k * 2^(j/32) * e^r, with 2^(j/32) from a 32-entry table (each entry correctly rounded; the
// tests recompute them) and e^r by its Taylor series through r^5 (truncation below 2.3e-15 relative).
// The integer n = 32 k + j is taken from the low mantissa bits of x * 32 / ln2 + 1.5 * 2^52, and the
// function has no branches, so a thread's independent calls overlap.  Arguments below -708 (and -inf
// and NaN) return 0: their terms are below 1e-307 next to a row maximum that contributes exactly 1.
// Written from the mathematics above; the polynomial coefficients are 1/k!.
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>

namespace jf {

#if defined(__CUDACC__)
#define JF_HD __host__ __device__ __forceinline__
#else
#define JF_HD inline
#endif

// 2^(j / 32) for j = 0 .. 31, each rounded to the nearest double.
#define JF_EXP2_FRAC32 { \
    0x1.0000000000000p+0, 0x1.059b0d3158574p+0, 0x1.0b5586cf9890fp+0, 0x1.11301d0125b51p+0, \
    0x1.172b83c7d517bp+0, 0x1.1d4873168b9aap+0, 0x1.2387a6e756238p+0, 0x1.29e9df51fdee1p+0, \
    0x1.306fe0a31b715p+0, 0x1.371a7373aa9cbp+0, 0x1.3dea64c123422p+0, 0x1.44e086061892dp+0, \
    0x1.4bfdad5362a27p+0, 0x1.5342b569d4f82p+0, 0x1.5ab07dd485429p+0, 0x1.6247eb03a5585p+0, \
    0x1.6a09e667f3bcdp+0, 0x1.71f75e8ec5f74p+0, 0x1.7a11473eb0187p+0, 0x1.82589994cce13p+0, \
    0x1.8ace5422aa0dbp+0, 0x1.93737b0cdc5e5p+0, 0x1.9c49182a3f090p+0, 0x1.a5503b23e255dp+0, \
    0x1.ae89f995ad3adp+0, 0x1.b7f76f2fb5e47p+0, 0x1.c199bdd85529cp+0, 0x1.cb720dcef9069p+0, \
    0x1.d5818dcfba487p+0, 0x1.dfc97337b9b5fp+0, 0x1.ea4afa2a490dap+0, 0x1.f50765b6e4540p+0 \
  }

// tab: the JF_EXP2_FRAC32 values (kernels keep a copy in shared memory)
JF_HD double exp_nonpos_f64(double x, const double* tab) {
  constexpr double kInvLn2x32 = 46.16624130844682;              // 32 / ln 2 (rounding only moves n by 1)
  constexpr double kLn2d32Hi = 0x1.62e42fee00000p-1 / 32.0;      // ln 2 / 32, 32 significant bits
  constexpr double kLn2d32Lo = 0x1.a39ef35793c76p-33 / 32.0;     // ln 2 / 32 - kLn2d32Hi
  constexpr double kShift = 0x1.8p52;
  const bool in_range = x >= -708.0;
  const double xc = in_range ? x : 0.0;
  const double t = fma(xc, kInvLn2x32, kShift);
  const double n = t - kShift;  // rint(32 x / ln 2), exact
  double r = fma(-n, kLn2d32Hi, xc);
  r = fma(-n, kLn2d32Lo, r);
  double p = 1.0 / 120.0;
  p = fma(p, r, 1.0 / 24.0);
  p = fma(p, r, 1.0 / 6.0);
  p = fma(p, r, 0.5);
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  int64_t tb;
#if defined(__CUDA_ARCH__)
  tb = __double_as_longlong(t);
#else
  std::memcpy(&tb, &t, sizeof(tb));
#endif
  const int ni = static_cast<int>(static_cast<uint32_t>(tb));  // n, in [-32704, 0]
  const int j = ni & 31;
  const int k = ni >> 5;  // floor(n / 32), in [-1022, 0]: 2^k is a normal double
  const int64_t bits = static_cast<int64_t>(k + 1023) << 52;
  double scale;
#if defined(__CUDA_ARCH__)
  scale = __longlong_as_double(bits);
#else
  std::memcpy(&scale, &bits, sizeof(scale));
#endif
  return in_range ? (tab[j] * p) * scale : 0.0;
}

}  // namespace jf
