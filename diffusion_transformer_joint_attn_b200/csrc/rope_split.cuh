// Rotary embedding of bf16 pairs to fp32, and the split of an fp32 value into
// two fp16 terms, for the compensated ("split") form of q~ k~^T.
//
// A rotated component a c - b s (or a s + b c), with a, b bf16 and c, s the
// fp32 table entries, has an exact value with up to ~60 significant bits.
// It is evaluated in fp64 (both products are exact there: 8 x 24 bits, the
// sum is rounded once) and rounded to fp32: r = RN32(RN64(a c - b s)).  r is
// then carried by two fp16 numbers, hi = RN16(r) and lo = RN16(r - hi) (the
// difference is exact in fp32), so hi + lo equals r to within 2^-22 |r| (or
// 2^-25 absolute where lo is an fp16 subnormal).  The tensor-core product
// hi_q.hi_k + hi_q.lo_k + lo_q.hi_k then carries q~.k~ to about 2^-21
// relative, where a single bf16 operand carries it to 2^-8.
// Inputs whose rotated magnitude exceeds the fp16 range (65504) are outside
// the contract of the split form.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace dit {

// The two rotated components of the bf16 pair packed in `w` (low half = even
// channel), each RN32(RN64(.)) of its exact value; without a table (rotate =
// false) the pair itself.
__device__ __forceinline__ float2 rotate_pair_f32(uint32_t w, float c, float s, bool rotate) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xFFFF0000u);
  if (!rotate) return make_float2(a, b);
  const double da = a, db = b;
  const double x = __fma_rn(da, static_cast<double>(c), -(db * static_cast<double>(s)));
  const double y = __fma_rn(da, static_cast<double>(s), db * static_cast<double>(c));
  return make_float2(__double2float_rn(x), __double2float_rn(y));
}

// hi = RN16(r), lo = RN16(r - hi) for the pair (r.x, r.y); each result packs
// the pair as fp16x2 (low half = even channel).
__device__ __forceinline__ void split_pair_f16(float2 r, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(r.x, r.y);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(r.x - hf.x, r.y - hf.y);   // both differences exact in fp32
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

}  // namespace dit
