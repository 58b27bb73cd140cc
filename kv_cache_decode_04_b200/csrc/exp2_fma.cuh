// exp2_fma.cuh -- 2^x evaluated on the FMA pipe, to take part of the softmax's
// exponentials off the special-function unit.
//
// Method: Cody-Waite range reduction, x = n + f with n the nearest integer
// (found by adding and subtracting 1.5 * 2^23) and |f| <= 1/2; 2^f by a
// degree-3 polynomial fitted by a Remez exchange for least maximum relative
// error on [-1/2, 1/2]; 2^n applied by adding n to the exponent field.  With
// the float32 coefficients below the relative error is below 1.5e-4 for
// -126 <= x <= 8 (softmax probabilities are rounded to bf16 afterwards, whose
// relative spacing is 2^-8).  Inputs below -126 are clamped there (result
// about 1e-38, never a wrapped exponent).
#pragma once

#define GQA_EXP2_C0 0.9999280571937561f
#define GQA_EXP2_C1 0.6932609677314758f
#define GQA_EXP2_C2 0.2426111251115799f
#define GQA_EXP2_C3 0.0551716685295105f

namespace gqa {

__device__ __forceinline__ float exp2_fma(float x) {
    x = fmaxf(x, -126.f);
    const float xr = x + 12582912.f;  // 1.5 * 2^23: the integer nearest x sits in the low mantissa bits
    const float f = x - (xr - 12582912.f);
    float p = fmaf(GQA_EXP2_C3, f, GQA_EXP2_C2);
    p = fmaf(p, f, GQA_EXP2_C1);
    p = fmaf(p, f, GQA_EXP2_C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(xr) << 23));
}

}  // namespace gqa
