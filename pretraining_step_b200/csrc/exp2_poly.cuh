// exp2_poly.cuh -- 2^x on the FMA pipe, for the share of the softmax
// exponentials that the attention backward takes off the exponential unit
// (MUFU ex2 delivers 16 results per clock per SM: one 128 x 128 score tile
// per 1024 clocks, as long as two 128 x 128 x 128 MMAs take).
//
// Method: range reduction x = n + f with n = rint(x), f in [-1/2, 1/2]
// (adding and subtracting the shifter 1.5 * 2^23 rounds to an integer and
// leaves n in the low bits of the sum), 2^f from a degree-3 polynomial, and
// n added to the exponent field of the result.  The polynomial is the
// minimax fit of the relative error on [-1/2, 1/2] found by the Remez
// exchange (exp2_poly_fit.py beside this package prints these constants):
// at most 7.5e-5 relative error, a twenty-sixth of bf16's half unit (2^-9),
// and the softmax rounds every probability to bf16.
#pragma once

#include <cuda_runtime.h>

namespace nc {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

// 2^x for two arguments with packed fp32 arithmetic.  x < 126; below -125
// the result is held near 2^-125 (not 0), so callers zero masked entries
// themselves; NaN gives that value too.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 sh = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
  const float2 t = __fadd2_rn(x, sh);                       // 1.5 * 2^23 + rint(x)
  const float2 nn = __ffma2_rn(t, make_float2(-1.f, -1.f), sh);  // -rint(x), exact
  const float2 f = __fadd2_rn(x, nn);                       // x - rint(x), exact
  float2 p = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  // The low bits of t hold rint(x) (two's complement, above 2^22 in the
  // mantissa); shifted by 23 they are exactly rint(x) << 23.
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace nc
