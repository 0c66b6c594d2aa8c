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
// Memory-bound: every thread owns 32 bytes of each part row (16 bf16 or 8
// fp32 channels: two 16-byte loads per part), so 8 (bf16 parts) or 16 (fp32
// parts) threads share a row; every load of a row, and those of the group's
// next row, are in flight at once;
// the parts are read through plain global loads, so they may live in a peer
// GPU's memory mapped into this context.
#include <cuda_bf16.h>

#include "launch.h"

namespace dit {
namespace {

constexpr int kThreads = 256;
// Channels of a row per thread, threads per row, rows per CTA.
template <bool kInF32>
constexpr int kChOf = kInF32 ? 8 : 16;
template <bool kInF32>
constexpr int kLanesOf = 128 / kChOf<kInF32>;
template <bool kInF32>
constexpr int kRowsOf = kThreads / kLanesOf<kInF32>;

struct MergeParams {
  const void* o[kMergeMaxParts];
  const float* lse[kMergeMaxParts];
  void* out;
  float* lse_out;
  long long rows;
  int R;
};

// The 32 bytes of one part row that this thread owns, as raw registers.
struct Chunk {
  uint4 w[2];
};

template <bool kInF32>
__device__ __forceinline__ Chunk load_chunk(const void* base, long long row, int sub) {
  const uint4* p = kInF32 ? reinterpret_cast<const uint4*>(static_cast<const float*>(base) + row * 128 + sub * 8)
                          : reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + row * 128 + sub * 16);
  Chunk c;
  c.w[0] = __ldg(p);
  c.w[1] = __ldg(p + 1);
  return c;
}

// The chunk's kChOf<kInF32> channels as fp32.
template <bool kInF32>
__device__ __forceinline__ void unpack(const Chunk& c, float* v) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(c.w);
  if (kInF32) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(u[e]);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v[2 * e] = __uint_as_float(u[e] << 16);
      v[2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
}

// One row's loads: R lses and R output chunks (parts past R read as empty).
template <int kR>
struct RowLoads {
  float l[kR];
  Chunk c[kR];
};

template <int kR, bool kInF32>
__device__ __forceinline__ void load_row(const MergeParams& p, long long row, int sub, RowLoads<kR>& x) {
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
  constexpr int kCh = kChOf<kInF32>;
  constexpr int kLanes = kLanesOf<kInF32>;
  constexpr int kRows = kRowsOf<kInF32>;
  const int sub = threadIdx.x % kLanes;
  const unsigned row_mask = ((1u << kLanes) - 1u) << (threadIdx.x & (32 - kLanes));
  const long long stride = static_cast<long long>(gridDim.x) * kRows;
  long long row = static_cast<long long>(blockIdx.x) * kRows + threadIdx.x / kLanes;
  RowLoads<kR> cur, nxt;
  if (kPrefetch) load_row<kR, kInF32>(p, row, sub, cur);
  for (; row < p.rows; row += stride) {
    if (kPrefetch)
      load_row<kR, kInF32>(p, row + stride, sub, nxt);
    else
      load_row<kR, kInF32>(p, row, sub, cur);
    const float* l = cur.l;
    const Chunk* c = cur.c;
    float m = -INFINITY;
#pragma unroll
    for (int r = 0; r < kR; ++r) m = fmaxf(m, l[r]);
    // every lane of the row has read the part lses before lse_out (which may
    // alias one of them) is written
    __syncwarp(row_mask);
    float acc[kCh];
#pragma unroll
    for (int e = 0; e < kCh; ++e) acc[e] = 0.f;
    float total = 0.f;
    const bool empty = m == -INFINITY;
    if (!empty) {
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        if (l[r] != -INFINITY) {      // an empty part's values are never used
          const float w = expf(l[r] - m);
          float v[kCh];
          unpack<kInF32>(c[r], v);
          total += w;
#pragma unroll
          for (int e = 0; e < kCh; ++e) acc[e] = fmaf(w, v[e], acc[e]);
        }
      }
      const float inv = 1.0f / total;
#pragma unroll
      for (int e = 0; e < kCh; ++e) acc[e] *= inv;
    }
    if (kOutF32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * 128 + sub * kCh);
#pragma unroll
      for (int i = 0; i < kCh / 4; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    } else {
      uint32_t w[kCh / 2];
#pragma unroll
      for (int e = 0; e < kCh / 2; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
        w[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row * 128 + sub * kCh);
#pragma unroll
      for (int i = 0; i < kCh / 8; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
    if (sub == 0 && p.lse_out != nullptr) p.lse_out[row] = empty ? -INFINITY : m + logf(total);
    if (kPrefetch) cur = nxt;
  }
}

// A grid-stride launch of the instance with exactly the CTAs that are
// resident at once (the rows are split evenly over them).
template <int kR, bool kInF32, bool kOutF32>
cudaError_t launch_one(const MergeParams& p, cudaStream_t s) {
  const long long need = (p.rows + kRowsOf<kInF32> - 1) / kRowsOf<kInF32>;
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
cudaError_t launch_bucket(const MergeParams& p, bool in_f32, bool out_f32, cudaStream_t s) {
  if (in_f32)
    return out_f32 ? launch_one<kR, true, true>(p, s) : launch_one<kR, true, false>(p, s);
  return out_f32 ? launch_one<kR, false, true>(p, s) : launch_one<kR, false, false>(p, s);
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
  if (a.R <= 2) return launch_bucket<2>(p, a.in_f32, a.out_f32, s);
  if (a.R <= 4) return launch_bucket<4>(p, a.in_f32, a.out_f32, s);
  if (a.R <= 8) return launch_bucket<8>(p, a.in_f32, a.out_f32, s);
  return launch_bucket<16>(p, a.in_f32, a.out_f32, s);
}

}  // namespace dit
