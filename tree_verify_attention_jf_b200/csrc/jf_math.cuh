// jf_math.cuh -- float64 exp for non-positive arguments, used for the draft-logit row sums.
//
// Method: Cody & Waite additive range reduction (W. J. Cody and W. Waite, "Software Manual for the
// Elementary Functions", 1980): x = n ln2 + r with n = rint(x / ln2) and |r| <= ln2 / 2, where ln2
// is split into a 32-bit head (so n * head is exact) and a tail; then e^r by its Taylor series
// through r^13 (truncation below 5e-18 relative for |r| <= 0.3466), evaluated in Horner form with
// fused multiply-adds; finally the exponent field is built from n.  Arguments below -708 return 0
// (their terms are below 1e-307 next to a row maximum that contributes exactly 1).  n is rounded with
// the 1.5 * 2^52 shift (the integer lands in the low mantissa bits), and the function has no
// branches, so a thread's independent calls overlap.
// Written from the mathematics above; the coefficients are 1/k!.
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

JF_HD double exp_nonpos_f64(double x) {
  constexpr double kInvLn2 = 1.4426950408889634;
  constexpr double kLn2Hi = 0x1.62e42fee00000p-1;  // ln 2 with its low 21 mantissa bits cleared
  constexpr double kLn2Lo = 0x1.a39ef35793c76p-33;  // ln 2 - kLn2Hi
  constexpr double kShift = 0x1.8p52;  // x / ln2 + kShift rounds x / ln2 to an integer in the low bits
  // Branch-free: out-of-range arguments (below -708, -inf, NaN) are computed as 0 and replaced at the end.
  const bool in_range = x >= -708.0;
  const double xc = in_range ? x : 0.0;
  const double t = fma(xc, kInvLn2, kShift);
  const double n = t - kShift;  // rint(x / ln2), exact
  double r = fma(-n, kLn2Hi, xc);
  r = fma(-n, kLn2Lo, r);
  double p = 1.0 / 6227020800.0;        // 1/13!
  p = fma(p, r, 1.0 / 479001600.0);     // 1/12!
  p = fma(p, r, 1.0 / 39916800.0);      // 1/11!
  p = fma(p, r, 1.0 / 3628800.0);       // 1/10!
  p = fma(p, r, 1.0 / 362880.0);        // 1/9!
  p = fma(p, r, 1.0 / 40320.0);         // 1/8!
  p = fma(p, r, 1.0 / 5040.0);          // 1/7!
  p = fma(p, r, 1.0 / 720.0);           // 1/6!
  p = fma(p, r, 1.0 / 120.0);           // 1/5!
  p = fma(p, r, 1.0 / 24.0);            // 1/4!
  p = fma(p, r, 1.0 / 6.0);             // 1/3!
  p = fma(p, r, 0.5);                   // 1/2!
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  // n in [-1022, 0] sits in the low 32 bits of t; 2^n is a normal double
  int64_t tb;
#if defined(__CUDA_ARCH__)
  tb = __double_as_longlong(t);
#else
  std::memcpy(&tb, &t, sizeof(tb));
#endif
  const int ni = static_cast<int>(static_cast<uint32_t>(tb));
  const int64_t bits = static_cast<int64_t>(ni + 1023) << 52;
  double scale;
#if defined(__CUDA_ARCH__)
  scale = __longlong_as_double(bits);
#else
  std::memcpy(&scale, &bits, sizeof(scale));
#endif
  return in_range ? p * scale : 0.0;
}

}  // namespace jf
