// x_rot = R(pos) x for bf16 x [B][H][N][D]: every channel pair turned by the
// table's (cos, sin) of its token and rounded exactly to bf16.  Memory-bound:
// each 16-byte chunk (4 pairs) is read once and written once; the table rows
// (N x 512 bytes) are shared by all B x H heads and stay in L2.
#include "launch.h"
#include <cuda_fp16.h>

#include "rope_exact.cuh"
#include "rope_split.cuh"

namespace dit {

__global__ void __launch_bounds__(256) rope_apply_kernel(const uint4* __restrict__ x, const float* __restrict__ tc,
                                                         const float* __restrict__ ts, uint4* __restrict__ y,
                                                         long long chunks, int N) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < chunks; c += stride) {
    const long long row = c >> 4;                 // 16 chunks of 8 channels per token row
    const int n = static_cast<int>(row % N);
    const int j0 = n * 64 + static_cast<int>(c & 15) * 4;
    const uint4 v = __ldg(x + c);
    const float4 cs = __ldg(reinterpret_cast<const float4*>(tc + j0));
    const float4 sn = __ldg(reinterpret_cast<const float4*>(ts + j0));
    uint4 o;
    o.x = rotate_pair_bf16(v.x, cs.x, sn.x);
    o.y = rotate_pair_bf16(v.y, cs.y, sn.y);
    o.z = rotate_pair_bf16(v.z, cs.z, sn.z);
    o.w = rotate_pair_bf16(v.w, cs.w, sn.w);
    y[c] = o;
  }
}

cudaError_t launch_rope_apply(const RopeApplyArgs& a, cudaStream_t s) {
  const long long chunks = static_cast<long long>(a.B) * a.H * a.N * (a.D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (chunks + 255) / 256;
  const long long cap = static_cast<long long>(sms) * 8;     // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  rope_apply_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<const uint4*>(a.x), a.cos, a.sin,
                                                                  static_cast<uint4*>(a.y), chunks, a.N);
  return cudaGetLastError();
}

// k_rot = R(pos) k (exactly rounded bf16) and v_f16 = fp16(v): the operands of
// the attention kernel's two MMAs, prepared once per call.  Chunks [0, C) are
// K, [C, 2C) are V.
__global__ void __launch_bounds__(256) prepare_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                         const float* __restrict__ tc, const float* __restrict__ ts,
                                                         uint4* __restrict__ k_rot, uint4* __restrict__ v_f16,
                                                         long long chunks, int N) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < 2 * chunks; c += stride) {
    if (c < chunks) {
      const long long row = c >> 4;
      const int n = static_cast<int>(row % N);
      const int j0 = n * 64 + static_cast<int>(c & 15) * 4;
      const uint4 x = __ldg(k + c);
      const float4 cs = __ldg(reinterpret_cast<const float4*>(tc + j0));
      const float4 sn = __ldg(reinterpret_cast<const float4*>(ts + j0));
      uint4 o;
      o.x = rotate_pair_bf16(x.x, cs.x, sn.x);
      o.y = rotate_pair_bf16(x.y, cs.y, sn.y);
      o.z = rotate_pair_bf16(x.z, cs.z, sn.z);
      o.w = rotate_pair_bf16(x.w, cs.w, sn.w);
      k_rot[c] = o;
    } else {
      const uint4 x = __ldg(v + (c - chunks));
      uint4 o;
      const uint32_t* w = &x.x;
      uint32_t* r = &o.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 h = __floats2half2_rn(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
        r[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      v_f16[c - chunks] = o;
    }
  }
}

cudaError_t launch_prepare_kv(const PrepareKVArgs& a, cudaStream_t s) {
  const long long chunks = static_cast<long long>(a.B) * a.H * a.N * (a.D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (2 * chunks + 255) / 256;
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  prepare_kv_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const uint4*>(a.k), static_cast<const uint4*>(a.v), a.cos, a.sin, static_cast<uint4*>(a.k_rot),
      static_cast<uint4*>(a.v_f16), chunks, a.N);
  return cudaGetLastError();
}

// The operands of the split (compensated) form of the attention's q~ k~^T:
// k_split[0] = hi, k_split[1] = lo of the fp32 rotated k (rope_split.cuh),
// each fp16 [B][H][N][D], and v_f16 = fp16(v).  Chunks [0, C) are K, [C, 2C)
// are V.  Without a table (tc == nullptr) k is split unrotated.
__global__ void __launch_bounds__(256)
    prepare_kv_split_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, const float* __restrict__ tc,
                            const float* __restrict__ ts, uint4* __restrict__ k_split, uint4* __restrict__ v_f16,
                            long long chunks, int N) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const bool rotate = tc != nullptr;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < 2 * chunks; c += stride) {
    if (c < chunks) {
      const uint4 x = __ldg(k + c);
      float4 cs = make_float4(1.f, 1.f, 1.f, 1.f), sn = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rotate) {
        const int n = static_cast<int>((c >> 4) % N);
        const int j0 = n * 64 + static_cast<int>(c & 15) * 4;
        cs = __ldg(reinterpret_cast<const float4*>(tc + j0));
        sn = __ldg(reinterpret_cast<const float4*>(ts + j0));
      }
      uint4 hi, lo;
      split_pair_f16(rotate_pair_f32(x.x, cs.x, sn.x, rotate), hi.x, lo.x);
      split_pair_f16(rotate_pair_f32(x.y, cs.y, sn.y, rotate), hi.y, lo.y);
      split_pair_f16(rotate_pair_f32(x.z, cs.z, sn.z, rotate), hi.z, lo.z);
      split_pair_f16(rotate_pair_f32(x.w, cs.w, sn.w, rotate), hi.w, lo.w);
      k_split[c] = hi;
      k_split[chunks + c] = lo;
    } else {
      const uint4 x = __ldg(v + (c - chunks));
      uint4 o;
      const uint32_t* w = &x.x;
      uint32_t* r = &o.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 h = __floats2half2_rn(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
        r[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      v_f16[c - chunks] = o;
    }
  }
}

cudaError_t launch_prepare_kv_split(const PrepareKVArgs& a, cudaStream_t s) {
  const long long chunks = static_cast<long long>(a.B) * a.H * a.N * (a.D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (2 * chunks + 255) / 256;
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  prepare_kv_split_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const uint4*>(a.k), static_cast<const uint4*>(a.v), a.cos, a.sin, static_cast<uint4*>(a.k_rot),
      static_cast<uint4*>(a.v_f16), chunks, a.N);
  return cudaGetLastError();
}

}  // namespace dit
