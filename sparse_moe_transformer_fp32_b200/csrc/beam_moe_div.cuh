// Correctly rounded FP32 division by a value shared by many dividends.
#pragma once

namespace beam {

// x / d rounded to nearest even for d > 0, given y = the correctly rounded 1 / d.
// q0 = RN(x y) can be more than an ulp from x / d, so one FMA correction
// q1 = RN(q0 + RN(x - d q0) y) first brings it within an ulp (its error is the second-order
// product of q0's and y's).  Then Markstein's theorem (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Develop. 34(1),
// 1990): for q1 within an ulp of x / d and y within half an ulp of 1 / d, the remainder
// x - d q1 is exactly representable (one FMA forms it) and RN(q1 + rem y) = RN(x / d).  The
// argument needs d, y and the quotient normal: callers take the plain division when d is
// below kDivRnMin or above kDivRnMax; the quotients here are bounded by a few hundred, and one
// that falls below the normal range rounds to a zero code either way.  A zero dividend keeps
// its sign, as in x / d.
constexpr float kDivRnMin = 1.0e-30f;
constexpr float kDivRnMax = 1.0e30f;

__device__ __forceinline__ bool div_rn_by_applies(float d) {
  return d >= kDivRnMin && d <= kDivRnMax;
}

__device__ __forceinline__ float div_rn_by(float x, float d, float y) {
  const float q0 = __fmul_rn(x, y);
  const float q1 = __fmaf_rn(__fmaf_rn(-d, q0, x), y, q0);
  const float q = __fmaf_rn(__fmaf_rn(-d, q1, x), y, q1);
  return x == 0.f ? x : q;
}

}  // namespace beam
