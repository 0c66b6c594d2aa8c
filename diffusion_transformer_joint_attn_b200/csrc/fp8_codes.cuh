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

// E4M3 codes of the correctly rounded fp32 quotients v[e] / scale of 8 values
// (code e in byte e % 4 of w0 (e < 4) or w1), from r = 1 / scale rounded to
// nearest (scale and r normal); false if some code is undecided, and then
// the caller divides.
//
// q = RN(v r) is within 3 fp32 ulps of the correctly rounded quotient: r and
// the product are each rounded once, with relative error at most 2^-24.
// E4M3 keeps 3 mantissa bits, so in its normal range (|q| >= 2^-6) the
// rounding midpoints are the fp32 values whose 20 low mantissa bits are
// 0x80000; rounding is monotonic, so q has the quotient's code unless a
// midpoint lies within those 3 ulps.  Decided: no q whose low 20 bits lie in
// 0x7FFF8 .. 0x80008 (within 8 units of the midpoint; their unsigned
// distance below 0x7FFF8 wraps above 16), and every q either an exact zero
// (its code is the quotient's, 0) or at least 2^-6 in magnitude.  Between
// 2^-6 and the subnormal codes the spacing changes but no midpoint lies near
// 2^-6 (the largest subnormal code is 7 x 2^-9); below 2^-6 the midpoints sit
// elsewhere, so such values leave the 8 undecided, as do ties.  Both tests
// are running unsigned minima over the 8 values.
__device__ __forceinline__ bool e4m3x8_of_quotients(const float* v, float r, uint32_t& w0, uint32_t& w1) {
  float q[8];
  uint32_t mag_min = 0xFFFFFFFFu, dist_min = 0xFFFFFFFFu;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    q[e] = v[e] * r;
    const uint32_t u = __float_as_uint(q[e]);
    mag_min = min(mag_min, (u & 0x7FFFFFFFu) - 1u);   // an exact zero wraps to the top
    dist_min = min(dist_min, (u & 0xFFFFFu) - 0x7FFF8u);
  }
  w0 = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
  w1 = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
  return mag_min >= 0x3C800000u - 1u && dist_min > 16u;   // 0x3C800000: 2^-6
}

// The same 8 codes through the IEEE division.
__device__ __forceinline__ void e4m3x8_by_division(const float* v, float scale, uint32_t& w0, uint32_t& w1) {
  float q[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) q[e] = __fdiv_rn(v[e], scale);
  w0 = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
  w1 = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
}

}  // namespace dit
