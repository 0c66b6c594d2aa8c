// FP8 E4M3 block quantisation of Q / K / V for the FP8 attention variant.
//
// One CTA per block of 64 tokens x 128 channels of one (b, h).  With rotary
// tables, each pair is first turned exactly as in fp64 with the fp32 table
// entries (x c - y s with both products exact, one rounding) and rounded to
// fp32.  The block's scale is amax / 448 in fp32 (1 for an all-zero block);
// each element becomes the E4M3 code of the fp32 quotient x / scale, rounded
// to nearest even and saturated to +-448.  The quotients come from one
// multiplication by the block's reciprocal scale whenever that decides the
// codes (e4m3x8_of_quotients, 8 at a time); the IEEE division runs only for
// the 8 values of a chunk with a quotient near an E4M3 rounding midpoint or
// nonzero below 2^-6.
#include <cuda_fp8.h>

#include "fp8_codes.cuh"
#include "launch.h"

namespace dit {
namespace {

constexpr int kBlockTokens = 64;
constexpr int kThreads = 256;
constexpr int kChunks = kBlockTokens * 128 / 8;         // 8 channels per chunk
constexpr int kPerThread = kChunks / kThreads;          // 4

// 16-byte streaming load: not kept in L1, and L2 fetches the 256-byte
// sector group around it (the neighbouring threads' chunks).
__device__ __forceinline__ uint4 ld_stream16(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <bool kRotate>
__device__ __forceinline__ void quantize_block(const uint4* __restrict__ x, const float* __restrict__ tc,
                                               const float* __restrict__ ts, uint2* __restrict__ codes,
                                               float* __restrict__ scales, int N, int blocks_per_bh) {
  __shared__ float warp_max[kThreads / 32];
  const int bh = blockIdx.x / blocks_per_bh;
  const int blk = blockIdx.x % blocks_per_bh;
  const int n0 = blk * kBlockTokens;
  float v[kPerThread][8];               // the thread's chunks as fp32 (rotated for q, k)
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int c = threadIdx.x + u * kThreads;
    const int n = n0 + (c >> 4);               // 16 chunks per token row
    if (n < N) {
      const uint4 w = ld_stream16(x + (static_cast<long long>(bh) * N + n) * 16 + (c & 15));
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      if constexpr (kRotate) {
        // the four pairs of this chunk: table entries n * 64 + (c & 15) * 4 + 0..3
        const float4 c4 = __ldg(reinterpret_cast<const float4*>(tc) + n * 16 + (c & 15));
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(ts) + n * 16 + (c & 15));
        const float cs[4] = {c4.x, c4.y, c4.z, c4.w}, sn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = __uint_as_float(ww[e] << 16), b = __uint_as_float(ww[e] & 0xFFFF0000u);
          v[u][2 * e] = rot_f64(a, cs[e], b, -sn[e]);
          v[u][2 * e + 1] = rot_f64(a, sn[e], b, cs[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[u][2 * e] = __uint_as_float(ww[e] << 16);
          v[u][2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[u][e]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  float bmax = warp_max[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) bmax = fmaxf(bmax, warp_max[w]);
  const float scale = bmax == 0.f ? 1.0f : __fdiv_rn(bmax, 448.0f);
  if (threadIdx.x == 0) scales[blockIdx.x] = scale;
  // the reciprocal path needs scale and 1 / scale normal: scale in [2^-126, 2^126]
  const bool via_reciprocal = scale >= 1.17549435e-38f && scale <= 8.50705917e+37f;
  const float r = __frcp_rn(scale);
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int c = threadIdx.x + u * kThreads;
    const int n = n0 + (c >> 4);
    if (n >= N) continue;
    uint32_t word[2];
    if (!via_reciprocal || !e4m3x8_of_quotients(v[u], r, word[0], word[1]))
      e4m3x8_by_division(v[u], scale, word[0], word[1]);
    codes[(static_cast<long long>(bh) * N + n) * 16 + (c & 15)] = make_uint2(word[0], word[1]);
  }
}

// 64 registers: 4 CTAs (32 warps, 64 KB of loads in flight) per SM.
__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint4* __restrict__ x, const float* __restrict__ tc,
                                                            const float* __restrict__ ts, uint2* __restrict__ codes,
                                                            float* __restrict__ scales, int N, int blocks_per_bh) {
  quantize_block<true>(x, tc, ts, codes, scales, N, blocks_per_bh);
}
__global__ void __launch_bounds__(kThreads)
    quantize_unrotated_kernel(const uint4* __restrict__ x, uint2* __restrict__ codes, float* __restrict__ scales, int N,
                              int blocks_per_bh) {
  quantize_block<false>(x, nullptr, nullptr, codes, scales, N, blocks_per_bh);
}

}  // namespace

cudaError_t launch_quantize_fp8(const QuantFp8Args& a, cudaStream_t s) {
  const int blocks_per_bh = (a.N + kBlockTokens - 1) / kBlockTokens;
  const long long grid = static_cast<long long>(a.B) * a.H * blocks_per_bh;
  if (a.cos != nullptr)
    quantize_kernel<<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const uint4*>(a.x), a.cos, a.sin, static_cast<uint2*>(a.codes), a.scale, a.N, blocks_per_bh);
  else
    quantize_unrotated_kernel<<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
        static_cast<const uint4*>(a.x), static_cast<uint2*>(a.codes), a.scale, a.N, blocks_per_bh);
  return cudaGetLastError();
}

}  // namespace dit
