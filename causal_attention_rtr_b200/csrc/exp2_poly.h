// exp2_poly.h -- 2^x on the FMA pipe, for part of the softmax exponentials.
//
// Method: Cody-Waite style range reduction for base 2 (x = n + f with n the
// nearest integer, f in [-0.5, 0.5]), a degree-3 polynomial for 2^f, and the
// exponent n added to the result's exponent field.  The polynomial is the
// minimax approximation of 2^f on [-0.5, 0.5] in relative error, computed for
// this library by the Remez exchange algorithm; its maximum relative error is
// 7.5e-5 (fp32 Horner evaluation), far below the 2^-9 rounding of the bf16
// probabilities it feeds.  n is taken with the round-to-nearest "magic
// number" addition 1.5 * 2^23.  Valid for finite x <= 64; inputs below -125
// are clamped (their result, < 2^-125, is negligible next to the row sum).
#pragma once

#include "ptx.cuh"   // ffma2, fadd2

#define RTR_EXP2_C0 0.9999280571937561f
#define RTR_EXP2_C1 0.6932609677314758f
#define RTR_EXP2_C2 0.2426111251115799f
#define RTR_EXP2_C3 0.0551716685295105f

namespace rtr {

__device__ __forceinline__ float exp2_poly(float x) {
    x = fmaxf(x, -125.0f);
    const float t = x + 12582912.0f;           // 1.5 * 2^23: low mantissa bits hold round(x)
    const float n = t - 12582912.0f;
    const float f = x - n;                      // [-0.5, 0.5]
    float p = fmaf(RTR_EXP2_C3, f, RTR_EXP2_C2);
    p = fmaf(p, f, RTR_EXP2_C1);
    p = fmaf(p, f, RTR_EXP2_C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// The same evaluation for two inputs at once: the reduction and the Horner
// steps as packed f32x2 instructions (half the FMA-pipe issue of two scalar
// calls), the clamp and the exponent insertion per element.  Results are
// identical to exp2_poly on each element.
__device__ __forceinline__ float2 exp2_poly_x2(float2 x) {
    x.x = fmaxf(x.x, -125.0f);
    x.y = fmaxf(x.y, -125.0f);
    const float2 magic = make_float2(12582912.0f, 12582912.0f);
    const float2 t = fadd2(x, magic);
    const float2 n = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);
    float2 p = ffma2(make_float2(RTR_EXP2_C3, RTR_EXP2_C3), f, make_float2(RTR_EXP2_C2, RTR_EXP2_C2));
    p = ffma2(p, f, make_float2(RTR_EXP2_C1, RTR_EXP2_C1));
    p = ffma2(p, f, make_float2(RTR_EXP2_C0, RTR_EXP2_C0));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace rtr
