// Correctly rounded rotary embedding of bf16 pairs.
//
// A pair (a, b) turns to (a c - b s, a s + b c) with fp32 table entries c, s;
// each component is returned as the bf16 nearest (ties to even) to its EXACT
// value.  A plain fp32 evaluation is off by up to ~1 fp32 ulp, which flips the
// bf16 rounding of about 1e-5 of all elements; on activation-outlier channels
// (|x| ~ 50) one such flip moves an attention logit by ~1.  So:
//  * fast path: bracket the exact value X between a round-down and a
//    round-up evaluation (directed-rounding mul and fma).  Rounding to bf16
//    is monotone, so if both ends round to the same bf16, so does X;
//  * otherwise (about 1e-4 of the pairs) rebuild X exactly as hi + lo from
//    error-free products (a c = p1 + e1 via fma) and Knuth's two-sum; lo
//    breaks the tie when hi sits exactly on a bf16 midpoint.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace dit {

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// fp32 value whose nearest-even bf16 is the bf16 nearest to the exact a*c + b*d.
__device__ __forceinline__ float dot2_exact_for_bf16(float a, float c, float b, float d) {
  const float p1 = __fmul_rn(a, c);
  const float e1 = __fmaf_rn(a, c, -p1);
  const float p2 = __fmul_rn(b, d);
  const float e2 = __fmaf_rn(b, d, -p2);
  const float h0 = __fadd_rn(p1, p2);
  const float z = __fsub_rn(h0, p1);
  const float err = __fadd_rn(__fsub_rn(p1, __fsub_rn(h0, z)), __fsub_rn(p2, z));
  const float l0 = __fadd_rn(err, __fadd_rn(e1, e2));
  const float hi = __fadd_rn(h0, l0);
  const float lo = __fsub_rn(l0, __fsub_rn(hi, h0));
  uint32_t u = __float_as_uint(hi);
  if ((u & 0xFFFFu) == 0x8000u && lo != 0.0f) u += ((lo > 0.0f) == (hi > 0.0f)) ? 1u : 0xFFFFFFFFu;
  return __uint_as_float(u);
}

// Exact path for one pair: (x, y) packed as bf16x2, low half = x.
static __device__ __noinline__ uint32_t rotate_pair_exact(float a, float b, float c, float s) {
  return pack_bf16x2_rn(dot2_exact_for_bf16(a, c, b, -s), dot2_exact_for_bf16(a, s, b, c));
}

// Rotate the bf16 pair packed in `w` (low half = even channel) by (c, s).
__device__ __forceinline__ uint32_t rotate_pair_bf16(uint32_t w, float c, float s) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xFFFF0000u);
  // x = a c - b s, y = a s + b c, each bracketed by directed roundings
  const float x_lo = __fmaf_rd(a, c, __fmul_rd(b, -s));
  const float x_hi = __fmaf_ru(a, c, __fmul_ru(b, -s));
  const float y_lo = __fmaf_rd(a, s, __fmul_rd(b, c));
  const float y_hi = __fmaf_ru(a, s, __fmul_ru(b, c));
  const uint32_t lo = pack_bf16x2_rn(x_lo, y_lo);
  const uint32_t hi = pack_bf16x2_rn(x_hi, y_hi);
  if (lo == hi) return lo;
  return rotate_pair_exact(a, b, c, s);
}

}  // namespace dit
