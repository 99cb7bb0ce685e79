// exp2 on the FMA pipe, for the share of softmax exponentials that would
// otherwise queue on the MUFU unit.
//
// Cody-Waite split 2^x = 2^j * 2^f with j = round(x) (added and subtracted
// 1.5 * 2^23, so j also sits in the low mantissa bits of the rounded value)
// and f = x - j in [-1/2, 1/2]; 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 with
// coefficients from exp2_poly_fit.py (Lawson minimax fit of the relative
// error, max 7.5e-5 on [-1/2, 1/2], far below the 2^-9 rounding of the bf16 P
// it feeds); 2^j is applied by adding j to the exponent field.  Inputs below
// -126 are clamped there (the exponent add then stays >= 0), giving a tiny positive value that rounds to zero in
// bf16 and is negligible in the fp32 row sum.
#pragma once

namespace dhsa {

__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23: rounds x to an integer
  const float j = t - 12582912.0f;
  const float f = x - j;
  float p = fmaf(5.517149398e-02f, f, 2.426109384e-01f);
  p = fmaf(p, f, 6.932609938e-01f);
  p = fmaf(p, f, 9.999280849e-01f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace dhsa
