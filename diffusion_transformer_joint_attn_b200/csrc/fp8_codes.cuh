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
// midpoint lies within those 3 ulps, i.e. unless q's low bits are within a
// few units of 0x80000 (tested as: bits 5-19 of q + 8 equal 0x80000, which
// flags 0x7FFF8 .. 0x80017).  Between 2^-6 and the subnormal codes the
// spacing changes but no midpoint lies near 2^-6 (the largest subnormal
// code is 7 x 2^-9); below 2^-6 the midpoints sit elsewhere, so such values
// (exact zeros included) leave the block undecided, as do ties.
__device__ __forceinline__ bool e4m3x8_of_quotients(const float* v, float r, uint32_t& w0, uint32_t& w1) {
  float q[8];
  float qmin = INFINITY;
  bool near_midpoint = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    q[e] = v[e] * r;
    qmin = fminf(qmin, fabsf(q[e]));
    near_midpoint |= ((__float_as_uint(q[e]) + 8u) & 0xFFFE0u) == 0x80000u;
  }
  w0 = e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
  w1 = e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16);
  return !near_midpoint && qmin >= 0.015625f;   // 2^-6
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
