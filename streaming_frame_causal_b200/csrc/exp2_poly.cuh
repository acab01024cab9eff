// exp2_poly.cuh -- 2^x for float pairs on the FMA/ALU pipes, used to take part
// of the softmax exponentials off the MUFU unit.
//
// Method: Cody-Waite style range reduction x = n + f with n = floor(x) and
// f in [0, 1), then 2^f by a cubic minimax (Remez exchange, relative error)
// polynomial evaluated in Horner form, and 2^n applied by adding n to the
// exponent field.  The coefficients were fitted for this library by
// exp2_poly_fit.py (next to this file): maximum relative error 7.5e-5 over
// [0, 1), well below the 2^-9 rounding of the bf16 probabilities it feeds.
//
// floor(x) comes from adding 1.5*2^23 with round-toward-minus-infinity: the sum
// is then the integer floor(x) + 1.5*2^23 exactly, and its low mantissa bits
// hold floor(x); shifting the sum's bit pattern left by 23 leaves exactly
// floor(x) << 23 (the constant's own bits vanish), ready to add to the
// polynomial's exponent.  The error bound holds for x >= -125 (below that the
// result turns denormal).  Inputs are clamped to [-126, +inf): the polynomial's
// exponent field is 126 or 127, so adding floor(x) << 23 never goes below zero
// (a clamp at -127 would wrap p(0) < 1 into the sign bit and give NaN); -inf
// (a masked score) therefore gives a value below 2^-125, zero for every purpose
// here.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace swa {

constexpr float kExp2C0 = 0.99992522f;
constexpr float kExp2C1 = 0.69583354f;
constexpr float kExp2C2 = 0.22606716f;
constexpr float kExp2C3 = 0.07802452f;
constexpr float kExp2Magic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rd(x, make_float2(kExp2Magic, kExp2Magic));      // floor(x) + magic
  const float2 fl = __fadd2_rn(t, make_float2(-kExp2Magic, -kExp2Magic));   // floor(x), exact
  const float2 f = __ffma2_rn(fl, make_float2(-1.f, -1.f), x);              // x - floor(x), exact
  float2 p = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  const uint32_t rx = __float_as_uint(p.x) + (__float_as_uint(t.x) << 23);
  const uint32_t ry = __float_as_uint(p.y) + (__float_as_uint(t.y) << 23);
  return make_float2(__uint_as_float(rx), __uint_as_float(ry));
}

}  // namespace swa
