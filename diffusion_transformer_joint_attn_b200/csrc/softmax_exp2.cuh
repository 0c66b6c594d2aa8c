// exp2 of softmax exponents on the FMA pipe, to share the work with the
// MUFU ex2 unit (whose 16 results per clock per SM tie the tensor-core rate
// of a 128 x 128 score tile).
//
// 2^x = 2^j * 2^f with j = rint(x) and |f| <= 1/2; 2^f comes from the
// degree-3 polynomial of least maximum RELATIVE error on [-1/2, 1/2]
// (7.5e-5 when evaluated in fp32, fitted by fit_exp2_poly.py in this
// directory: below the half-ulp 2^-12 of fp16, the format P is stored in;
// degree 4, at 2.6e-6, costs one more fused multiply-add pair per value
// pair), 2^j is added to the exponent field.  x is clamped to >= -125
// (results that small underflow fp16, the format P is stored in, anyway); the
// polynomial's value lies in [0.70, 1.42] (2^+-1/2 within its error), so its
// exponent field is 126 or 127 and adding j >= -125 leaves a field >= 1: the result is always the
// normal fp32 number p * 2^j.
// Operates on pairs with Blackwell's packed fp32 add / fma.
#pragma once

#include <cstdint>

namespace dit {

constexpr float kExp2C0 = 9.999280273e-01f;
constexpr float kExp2C1 = 6.932609466e-01f;
constexpr float kExp2C2 = 2.426113821e-01f;
constexpr float kExp2C3 = 5.517187452e-02f;
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23: x + magic holds rint(x) in its low mantissa bits

__device__ __forceinline__ void exp2_pair_poly(float x0, float x1, float& y0, float& y1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  uint32_t t0, t1;
  float p0, p1;
  asm("{\n\t.reg .b64 x, m, t, j, f, p, c;\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "mov.b64 m, {%6, %6};\n\t"
      "add.rn.f32x2 t, x, m;\n\t"          // t = x + magic (rint in the low bits)
      "sub.rn.f32x2 j, t, m;\n\t"          // j = rint(x)
      "sub.rn.f32x2 f, x, j;\n\t"          // f = x - j, |f| <= 1/2, exact
      "mov.b64 c, {%7, %7};\n\t"
      "mov.b64 p, {%8, %8};\n\t"
      "fma.rn.f32x2 p, p, f, c;\n\t"       // c3 f + c2
      "mov.b64 c, {%9, %9};\n\t"
      "fma.rn.f32x2 p, p, f, c;\n\t"       // (..) f + c1
      "mov.b64 c, {%10, %10};\n\t"
      "fma.rn.f32x2 p, p, f, c;\n\t"       // (..) f + c0
      "mov.b64 {%0, %1}, t;\n\t"
      "mov.b64 {%2, %3}, p;\n\t}"
      : "=r"(t0), "=r"(t1), "=f"(p0), "=f"(p1)
      : "f"(x0), "f"(x1), "f"(kRoundMagic), "f"(kExp2C2), "f"(kExp2C3), "f"(kExp2C1), "f"(kExp2C0));
  // 2^j: add j to the exponent field (the magic's own bits shift out)
  y0 = __uint_as_float(__float_as_uint(p0) + (t0 << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (t1 << 23));
}

}  // namespace dit
