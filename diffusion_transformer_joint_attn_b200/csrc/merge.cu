// Merge of partial attention results over disjoint key sets.
//
// When the keys of a row are split over R parts (context parallelism:
// wavespeed.ai "Beschleunigung der FLUX.1-dev Bildgenerierung", section on
// context parallelism and First Block Cache), part r returns its normalised
// output O_r and its log-sum-exp lse_r, and the result over the union is
//     lse = log sum_r exp(lse_r),   O = sum_r exp(lse_r - lse) O_r.
// A part with no keys has lse_r = -inf: its weight is 0 and the values of
// its O_r are not used; a row whose parts are all empty gets O = 0 and lse = -inf.
//
// Memory-bound: 16 threads per row, 8 channels (one 16-byte bf16 or two
// 16-byte fp32 loads per part) each, every load of a row in flight at once;
// the parts are read through plain global loads, so they may live in a peer
// GPU's memory mapped into this context.
#include <cuda_bf16.h>

#include "launch.h"

namespace dit {
namespace {

constexpr int kThreads = 256;
constexpr int kLanesPerRow = 16;
constexpr int kRowsPerBlock = kThreads / kLanesPerRow;

struct MergeParams {
  const void* o[kMergeMaxParts];
  const float* lse[kMergeMaxParts];
  void* out;
  float* lse_out;
  long long rows;
  int R;
};

// The 8 channels of one part row that this thread owns, as raw registers.
template <bool kInF32>
struct Chunk {
  uint4 w[kInF32 ? 2 : 1];
};

template <bool kInF32>
__device__ __forceinline__ Chunk<kInF32> load_chunk(const void* base, long long row, int sub) {
  Chunk<kInF32> c;
  if (kInF32) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + row * 128 + sub * 8);
    c.w[0] = __ldg(p);
    c.w[kInF32 ? 1 : 0] = __ldg(p + 1);
  } else {
    c.w[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + row * 128 + sub * 8));
  }
  return c;
}

template <bool kInF32>
__device__ __forceinline__ void unpack(const Chunk<kInF32>& c, float* v) {
  if (kInF32) {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(c.w);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(u[e]);
  } else {
    const uint32_t ww[4] = {c.w[0].x, c.w[0].y, c.w[0].z, c.w[0].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(ww[e] << 16);
      v[2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
    }
  }
}

// kR: parts this instantiation holds in registers (R <= kR).  All loads of a
// row (R lses, R output chunks) are issued before the first is used.
template <int kR, bool kInF32, bool kOutF32>
__global__ void __launch_bounds__(kThreads) merge_kernel(const MergeParams p) {
  const int sub = threadIdx.x % kLanesPerRow;
  const unsigned half_mask = 0xFFFFu << (threadIdx.x & 16);
  const long long stride = static_cast<long long>(gridDim.x) * kRowsPerBlock;
  for (long long row = static_cast<long long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kLanesPerRow;
       row < p.rows; row += stride) {
    float l[kR];
    Chunk<kInF32> c[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      if (r < p.R) {
        l[r] = __ldg(p.lse[r] + row);
        c[r] = load_chunk<kInF32>(p.o[r], row, sub);
      } else {
        l[r] = -INFINITY;
      }
    }
    float m = -INFINITY;
#pragma unroll
    for (int r = 0; r < kR; ++r) m = fmaxf(m, l[r]);
    // every lane of the row has read the part lses before lse_out (which may
    // alias one of them) is written
    __syncwarp(half_mask);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float total = 0.f;
    const bool empty = m == -INFINITY;
    if (!empty) {
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        if (l[r] != -INFINITY) {      // an empty part's values are never used
          const float w = expf(l[r] - m);
          float v[8];
          unpack<kInF32>(c[r], v);
          total += w;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, v[e], acc[e]);
        }
      }
      const float inv = 1.0f / total;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= inv;
    }
    if (kOutF32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * 128 + sub * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
        w[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row * 128 + sub * 8) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (sub == 0 && p.lse_out != nullptr) p.lse_out[row] = empty ? -INFINITY : m + logf(total);
  }
}

template <int kR>
void launch_bucket(const MergeParams& p, bool in_f32, bool out_f32, unsigned grid, cudaStream_t s) {
  if (in_f32) {
    if (out_f32)
      merge_kernel<kR, true, true><<<grid, kThreads, 0, s>>>(p);
    else
      merge_kernel<kR, true, false><<<grid, kThreads, 0, s>>>(p);
  } else {
    if (out_f32)
      merge_kernel<kR, false, true><<<grid, kThreads, 0, s>>>(p);
    else
      merge_kernel<kR, false, false><<<grid, kThreads, 0, s>>>(p);
  }
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s) {
  MergeParams p;
  for (int r = 0; r < kMergeMaxParts; ++r) {
    p.o[r] = r < a.R ? a.o[r] : nullptr;
    p.lse[r] = r < a.R ? a.lse[r] : nullptr;
  }
  p.out = a.out;
  p.lse_out = a.lse_out;
  p.rows = a.rows;
  p.R = a.R;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long need = (a.rows + kRowsPerBlock - 1) / kRowsPerBlock;
  const long long cap = static_cast<long long>(sms) * (2048 / kThreads);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  if (a.R <= 2)
    launch_bucket<2>(p, a.in_f32, a.out_f32, grid, s);
  else if (a.R <= 4)
    launch_bucket<4>(p, a.in_f32, a.out_f32, grid, s);
  else if (a.R <= 8)
    launch_bucket<8>(p, a.in_f32, a.out_f32, grid, s);
  else
    launch_bucket<16>(p, a.in_f32, a.out_f32, grid, s);
  return cudaGetLastError();
}

}  // namespace dit
