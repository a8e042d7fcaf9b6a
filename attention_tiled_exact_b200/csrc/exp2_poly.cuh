// 2^x on the FMA pipe, for a pair of inputs (the prefill kernel sends a share
// of its exponentials here because the MUFU unit is its scarce resource).
//
// Range reduction rounds x to the nearest integer n by adding 1.5 * 2^23 (the
// integer lands in the low mantissa bits; ties go to the even integer), so
// x = n + f with |f| <= 1/2. 2^f comes from a cubic fitted for this kernel by
// Lawson's iteratively reweighted least squares, minimising the relative error
// on [-1/2, 1/2] (attention_tiled_exact_b200/exp2_poly_fit.py computes the
// four coefficients; their maximum relative error is 7.48e-5, far below the 2^-9
// rounding of the bf16 P they feed). n is then added to the exponent field as
// an integer. Inputs are clamped at -126, so tiny results come out as about
// 2^-126 instead of 0 (below 2^-125 they are not accurate, only tiny), and
// inputs must stay below 128.
#pragma once

#include <cuda_runtime.h>

namespace attn {

// Coefficients of 2^f ~ C0 + C1 f + C2 f^2 + C3 f^3 (float32, from exp2_poly_fit.py).
constexpr float EXP2_C0 = 0.9999280571937561f;
constexpr float EXP2_C1 = 0.6932609677314758f;
constexpr float EXP2_C2 = 0.24261116981506348f;
constexpr float EXP2_C3 = 0.0551716648042202f;

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
  p = __ffma2_rn(p, f, make_float2(EXP2_C1, EXP2_C1));
  p = __ffma2_rn(p, f, make_float2(EXP2_C0, EXP2_C0));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace attn
