// FP8 E4M3 block quantisation of Q / K / V for the FP8 attention variant.
//
// One CTA per block of 64 tokens x 128 channels of one (b, h).  With rotary
// tables, each pair is first turned exactly as in fp64 with the fp32 table
// entries (x c - y s with both products exact, one rounding) and rounded to
// fp32.  The block's scale is amax / 448 in fp32 (1 for an all-zero block);
// each element becomes the E4M3 code of the fp32 quotient x / scale, rounded
// to nearest even and saturated to +-448.
#include <cuda_fp8.h>

#include "launch.h"

namespace dit {
namespace {

constexpr int kBlockTokens = 64;
constexpr int kThreads = 256;
constexpr int kChunks = kBlockTokens * 128 / 8;         // 8 channels per chunk
constexpr int kPerThread = kChunks / kThreads;          // 4

__device__ __forceinline__ float rot_f64(float a, float c, float b, float d) {
  // a c + b d with exact products, rounded once to fp64, then to fp32
  const double bd = static_cast<double>(b) * static_cast<double>(d);
  return static_cast<float>(fma(static_cast<double>(a), static_cast<double>(c), bd));
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint4* __restrict__ x, const float* __restrict__ tc,
                                                            const float* __restrict__ ts, uint2* __restrict__ codes,
                                                            float* __restrict__ scales, int N, int blocks_per_bh) {
  __shared__ float warp_max[kThreads / 32];
  const int bh = blockIdx.x / blocks_per_bh;
  const int blk = blockIdx.x % blocks_per_bh;
  const int n0 = blk * kBlockTokens;
  float v[kPerThread][8];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int c = threadIdx.x + u * kThreads;
    const int r = c >> 4;                      // 16 chunks per token row
    const int n = n0 + r;
    if (n < N) {
      const long long idx = (static_cast<long long>(bh) * N + n) * 16 + (c & 15);
      const uint4 w = __ldg(x + idx);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = __uint_as_float(ww[e] << 16), b = __uint_as_float(ww[e] & 0xFFFF0000u);
        if (tc != nullptr) {
          const int j = n * 64 + (c & 15) * 4 + e;
          const float cs = __ldg(tc + j), sn = __ldg(ts + j);
          v[u][2 * e] = rot_f64(a, cs, b, -sn);
          v[u][2 * e + 1] = rot_f64(a, sn, b, cs);
        } else {
          v[u][2 * e] = a;
          v[u][2 * e + 1] = b;
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
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int c = threadIdx.x + u * kThreads;
    const int n = n0 + (c >> 4);
    if (n >= N) continue;
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t two = e4m3x2(__fdiv_rn(v[u][2 * e], scale), __fdiv_rn(v[u][2 * e + 1], scale));
      if (e < 2)
        lo |= two << (16 * e);
      else
        hi |= two << (16 * (e - 2));
    }
    codes[(static_cast<long long>(bh) * N + n) * 16 + (c & 15)] = make_uint2(lo, hi);
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const QuantFp8Args& a, cudaStream_t s) {
  const int blocks_per_bh = (a.N + kBlockTokens - 1) / kBlockTokens;
  const long long grid = static_cast<long long>(a.B) * a.H * blocks_per_bh;
  quantize_kernel<<<static_cast<unsigned>(grid), kThreads, 0, s>>>(static_cast<const uint4*>(a.x), a.cos, a.sin,
                                                                   static_cast<uint2*>(a.codes), a.scale, a.N,
                                                                   blocks_per_bh);
  return cudaGetLastError();
}

}  // namespace dit
