// 2^x evaluated on the FMA and integer pipes instead of the special-function
// unit, so that a kernel whose exponentials saturate that unit can move part
// of them elsewhere (the published idea of splitting softmax exponentials
// between the MUFU and a polynomial on the FMA units, as in FlashAttention's
// Blackwell kernels; the polynomial and its coefficients here are our own).
//
// 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]:
//  * j: adding 1.5 * 2^23 rounds x to an integer held in the low mantissa
//    bits of the sum (round to nearest even, exact for |x| < 2^22);
//  * 2^f: a cubic in Horner form, interpolating 2^f at the four Chebyshev
//    nodes of [-1/2, 1/2] (coefficients from fit_exp2_poly.py); relative
//    error below 1.0e-4 in float32, under the rounding of the 16-bit P it
//    feeds;
//  * 2^j: j is added to the exponent field.  Shifting the sum's bits left by
//    23 leaves exactly j << 23 (the constant's own bits shift out).
// x is clamped below at -125 so the result stays a normal float (2^-125 is
// zero for every purpose here, and -inf maps to it); valid for x < 127.
#pragma once

#include <stdint.h>

namespace pa {

constexpr float kExp2C0 = 0.9999245405197144f;
constexpr float kExp2C1 = 0.6931367516517639f;
constexpr float kExp2C2 = 0.2426394820213318f;
constexpr float kExp2C3 = 0.05583828315138817f;
constexpr float kExp2Round = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + kExp2Round;
  const float f = x - (t - kExp2Round);
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// The same polynomial for two inputs, with the floating-point steps done as
// packed fp32x2 operations (sm_100: one instruction for both lanes; each lane
// rounds exactly as the scalar version does, so the results are identical).
__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float x0, float x1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  uint32_t t0, t1, p0, p1;
  asm("{\n\t"
      ".reg .b64 x, t, r, f, p, k;\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "mov.b64 k, {%6, %6};\n\t"
      "add.rn.f32x2 t, x, k;\n\t"       // t = x + 1.5 * 2^23
      "sub.rn.f32x2 r, t, k;\n\t"       // r = round(x)
      "sub.rn.f32x2 f, x, r;\n\t"       // f = x - round(x)
      "mov.b64 k, {%7, %7};\n\t"
      "mov.b64 p, {%8, %8};\n\t"
      "fma.rn.f32x2 p, k, f, p;\n\t"    // c3 f + c2
      "mov.b64 k, {%9, %9};\n\t"
      "fma.rn.f32x2 p, p, f, k;\n\t"    // (.) f + c1
      "mov.b64 k, {%10, %10};\n\t"
      "fma.rn.f32x2 p, p, f, k;\n\t"    // (.) f + c0
      "mov.b64 {%0, %1}, t;\n\t"
      "mov.b64 {%2, %3}, p;\n\t"
      "}"
      : "=r"(t0), "=r"(t1), "=r"(p0), "=r"(p1)
      : "f"(x0), "f"(x1), "f"(kExp2Round), "f"(kExp2C3), "f"(kExp2C2), "f"(kExp2C1), "f"(kExp2C0));
  y0 = __int_as_float(static_cast<int>(p0 + (t0 << 23)));
  y1 = __int_as_float(static_cast<int>(p1 + (t1 << 23)));
}

}  // namespace pa
