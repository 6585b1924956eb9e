// 2^x on the FMA pipe, used for part of the softmax exponentials so that the
// special-function unit is not the only producer of them.
//
// 2^x = 2^n * 2^f with n = floor(x), f = x - n in [0, 1). 2^f comes from a
// cubic in Horner form whose coefficients were fitted here to minimise the
// maximum relative error over [0, 1) (iteratively reweighted least squares
// on 20001 points, then rounded to fp32): max relative error 7.6e-5 in fp32
// evaluation, far below the bf16 rounding (2^-9) applied to P afterwards.
// 2^n is applied by adding n to the exponent field. Inputs below -126 give
// exactly 0 (masked logits are -inf).
#pragma once

namespace dfs {

constexpr float kExp2C0 = 0.9999262690544128f;
constexpr float kExp2C1 = 0.6958271861076355f;
constexpr float kExp2C2 = 0.22607102990150452f;
constexpr float kExp2C3 = 0.07802802324295044f;

__device__ __forceinline__ float exp2_poly(float x) {
  const float xc = fmaxf(x, -126.0f);
  const float n = floorf(xc);
  const float f = xc - n;
  float p = fmaf(kExp2C3, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
  const int bits = __float_as_int(p) + (static_cast<int>(n) << 23);
  return x < -126.0f ? 0.0f : __int_as_float(bits);
}

}  // namespace dfs
