// Correctly rounded fp32 quotients x / s for a divisor shared by many dividends:
// the quantisers divide every value of a frame, slot or block by one scale, and the
// quotient decides an e4m3 / e2m1 code, so it has to be the IEEE round-to-nearest
// quotient bit for bit.
//
// Method (Markstein's correction step, P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990;
// also the Handbook of Floating-Point Arithmetic, the division chapter): with
// y = RN(1/s) and a quotient q within one ulp of x/s, the residual r = x - s*q is
// exact when computed by one FMA, and RN(q + r*y) = RN(x/s).  The first estimate
// RN(x*y) can be up to 1.5 ulps off, so the step is applied twice: after the first
// the estimate is within half an ulp plus a 2^-24 fraction of one, which meets the
// premise of the second.  Five FMA-pipe operations per quotient, no branch.
//
// Range: the step needs the residual to stay a normal number wherever the quotient
// decides a code.  Codes are decided for |x/s| >= 2^-11 (e4m3 rounds anything
// smaller to zero; e2m1 anything below 0.25), where |x| >= 2^-11 * s; with
// s >= 2^-60 the residual (about 2^-24 |x|) is then >= 2^-95, far from the subnormal
// range.  Divisors below 2^-60, or not finite, take the IEEE division instead; the
// sign of a zero quotient is taken from the dividend, as IEEE division gives it.
#pragma once
#include <cuda_runtime.h>

namespace ckv {

struct SharedDivisor {
  float s, y;
  bool exact_path;  // true: use the IEEE division (divisor outside the step's range)
};

__device__ __forceinline__ SharedDivisor make_divisor(float s) {
  SharedDivisor d;
  d.s = s;
  d.exact_path = !(s >= 0x1p-60f) || !(s < 0x1p+120f);
  d.y = d.exact_path ? 1.0f : __frcp_rn(s);
  return d;
}

__device__ __forceinline__ float div_rn(float x, const SharedDivisor& d) {
  if (d.exact_path) return __fdiv_rn(x, d.s);
  float q = __fmul_rn(x, d.y);
  float r = __fmaf_rn(-q, d.s, x);
  q = __fmaf_rn(r, d.y, q);
  r = __fmaf_rn(-q, d.s, x);
  q = __fmaf_rn(r, d.y, q);
  return copysignf(q, x);
}

}  // namespace ckv
