// E4M3 ("e4m3fn": bias 7, largest finite 448, no infinities) codes of
// fp32 quotients x / scale, and the fp64-exact rotation of a pair, shared by
// the block quantiser (quant_fp8.cu) and the projection epilogue
// (qkv_proj.cu).
#pragma once

#include <cstdint>

namespace dit {

__device__ __forceinline__ float rot_f64(float a, float c, float b, float d) {
  // a c + b d with exact products, rounded once to fp64, then to fp32
  const double bd = static_cast<double>(b) * static_cast<double>(d);
  return static_cast<float>(fma(static_cast<double>(a), static_cast<double>(c), bd));
}

// E4M3 codes of lo (low byte) and hi (high byte), nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// E4M3 code of the correctly rounded fp32 quotient x / scale from
// r = 1 / scale rounded to nearest (scale and r normal); false if undecided.
// x * r is within 3 fp32 ulps of that quotient: r and the product are each
// rounded once, with relative error at most 2^-24.  Rounding to E4M3 is
// monotonic, so when the fp32 values 8 ulps below and above x * r (the lower
// magnitude clamped at 0) have one code, the quotient has it too.  They
// differ when the quotient lies within a few ulps of an E4M3 rounding
// midpoint (or is not finite); the caller then divides.
__device__ __forceinline__ bool e4m3_of_quotient(float x, float r, uint32_t& code) {
  const uint32_t u = __float_as_uint(x * r);
  const uint32_t mag = u & 0x7FFFFFFFu;
  const float below = __uint_as_float((u & 0x80000000u) | (max(mag, 8u) - 8u));
  const float above = __uint_as_float(u + 8u);
  const uint32_t two = e4m3x2(below, above);
  code = two & 0xFFu;
  return ((two ^ (two >> 8)) & 0xFFu) == 0u;
}

}  // namespace dit
