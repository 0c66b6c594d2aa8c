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
// 16-byte fp32 loads per part) each; every load of a row, and those of the
// group's next row, are in flight at once;
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

// One row's loads: R lses and R output chunks (parts past R read as empty).
template <int kR, bool kInF32>
struct RowLoads {
  float l[kR];
  Chunk<kInF32> c[kR];
};

template <int kR, bool kInF32>
__device__ __forceinline__ void load_row(const MergeParams& p, long long row, int sub, RowLoads<kR, kInF32>& x) {
#pragma unroll
  for (int r = 0; r < kR; ++r) {
    if (r < p.R && row < p.rows) {
      x.l[r] = __ldg(p.lse[r] + row);
      x.c[r] = load_chunk<kInF32>(p.o[r], row, sub);
    } else {
      x.l[r] = -INFINITY;
    }
  }
}

// kR: parts this instantiation holds in registers (R <= kR).  All loads of a
// row (R lses, R output chunks) are issued before the first is used; with up
// to 4 parts the loads of the group's next row are issued too before this
// row is combined (with more parts the registers would spill).
template <int kR, bool kInF32, bool kOutF32>
__global__ void __launch_bounds__(kThreads) merge_kernel(const MergeParams p) {
  constexpr bool kPrefetch = kR <= 4;
  const int sub = threadIdx.x % kLanesPerRow;
  const unsigned half_mask = 0xFFFFu << (threadIdx.x & 16);
  const long long stride = static_cast<long long>(gridDim.x) * kRowsPerBlock;
  long long row = static_cast<long long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kLanesPerRow;
  RowLoads<kR, kInF32> cur, nxt;
  if (kPrefetch) load_row<kR, kInF32>(p, row, sub, cur);
  for (; row < p.rows; row += stride) {
    if (kPrefetch)
      load_row<kR, kInF32>(p, row + stride, sub, nxt);
    else
      load_row<kR, kInF32>(p, row, sub, cur);
    const float* l = cur.l;
    const Chunk<kInF32>* c = cur.c;
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
    if (kPrefetch) cur = nxt;
  }
}

// A grid-stride launch of the instance with exactly the CTAs that are
// resident at once (the rows are split evenly over them).
template <int kR, bool kInF32, bool kOutF32>
cudaError_t launch_one(const MergeParams& p, long long need, cudaStream_t s) {
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const cudaError_t r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, merge_kernel<kR, kInF32, kOutF32>,
                                                                      kThreads, 0);
  if (r != cudaSuccess) return r;
  const long long cap = static_cast<long long>(sms) * (per_sm > 0 ? per_sm : 1);
  merge_kernel<kR, kInF32, kOutF32><<<static_cast<unsigned>(need < cap ? need : cap), kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <int kR>
cudaError_t launch_bucket(const MergeParams& p, bool in_f32, bool out_f32, long long need, cudaStream_t s) {
  if (in_f32)
    return out_f32 ? launch_one<kR, true, true>(p, need, s) : launch_one<kR, true, false>(p, need, s);
  return out_f32 ? launch_one<kR, false, true>(p, need, s) : launch_one<kR, false, false>(p, need, s);
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
  const long long need = (a.rows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (a.R <= 2) return launch_bucket<2>(p, a.in_f32, a.out_f32, need, s);
  if (a.R <= 4) return launch_bucket<4>(p, a.in_f32, a.out_f32, need, s);
  if (a.R <= 8) return launch_bucket<8>(p, a.in_f32, a.out_f32, need, s);
  return launch_bucket<16>(p, a.in_f32, a.out_f32, need, s);
}

}  // namespace dit
