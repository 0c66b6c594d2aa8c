// The QKV projection of the joint token sequence with the FP8 operand
// preparation fused into its epilogue (sm_100a).
//
//   y[b, n, o] = sum_c x[b, n, c] w[o, c] (+ bias[o]),  o = s H D + h D + d
//
// is a bf16 x bf16 -> fp32 GEMM on the tensor cores (tcgen05, accumulator
// in tensor memory).  Its epilogue turns the accumulator tile straight into
// the operands of dit_attn_forward_fp8, with no round trip of y through
// HBM: for q and k it applies the rotary embedding (each pair turned in
// fp64 from the fp32 accumulator and the fp32 table entries, rounded to
// fp32), takes the amax of every block of 64 tokens x 128 channels of one
// (b, h), and writes the E4M3 codes of y / (amax / 448) and the block scale;
// optionally also the unrotated y rounded to bf16 in the attention layout.
//
// CTA pairs (clusters of two) compute tiles of 256 tokens of one batch item
// (128 per CTA) x 256 output features (two heads); blockIdx.x runs over the
// feature tiles, so the pairs resident at once share their token rows of x and
// sweep the weight, most of which (57 MB at the FLUX width) is then read from
// L2, while x is read from HBM about once.  Per CTA, warp 0 loads x and w tiles
// of 64 input channels by TMA into a 3-stage ring, warp 1 (even CTA) issues the
// pair MMAs (M = 256, N = 256, K = 16 per instruction), and warps 2-9 run the
// epilogue in two groups of four (one thread per token row in each, lanes by
// warp & 3), one head each: a first pass over the accumulator for the block
// maxima, a second for the codes.  The two 64-token blocks of a CTA's tile are
// rows 0-63 (lane quarters 0-1) and 64-127 (quarters 2-3).  Two CTAs share an
// SM (96 KB of shared memory and 256 tensor-memory columns each), so one's
// epilogue runs while the other's MMAs do.
#include <cuda_bf16.h>

#include "fp8_codes.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "rope_exact.cuh"

namespace dit {
namespace {

constexpr int kBM = 128;                   // tokens per tile
constexpr int kBK = 64;                    // input channels per stage (one 128-byte swizzle row)
constexpr int kABytes = kBM * kBK * 2;     // 16 KB
constexpr int kThreads = 320;              // producer, MMA issuer, two epilogue warp groups
constexpr int kEpiThreads = 128;           // per epilogue warp group
constexpr int kBarEpi = 1;                 // named barriers 1 and 2, one per epilogue warp group

struct Params {
  const float* bias;        // [3 H D] or nullptr
  const float* cos;         // [N][64] or nullptr
  const float* sin;
  uint8_t* codes[3];        // q8, k8, v8: [B][H][N][128]
  float* scales[3];         // [B][H][ceil(N/64)]
  __nv_bfloat16* y16[3];    // optional bf16 q, k, v [B][H][N][128] (nullptr: not written)
  int* status;
  int N, C, H;
  int k_steps;
};

// The 32 accumulator columns at taddr of this thread's row (a warp-collective
// load: every lane calls it), plus the bias of those columns (shared memory): y.
__device__ __forceinline__ void load_y(uint32_t taddr, const float* bias32, float* y) {
  uint32_t u[32];
  tmem_ld32(taddr, u);
  tmem_ld_wait(u);
  const float4* b4 = reinterpret_cast<const float4*>(bias32);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 bb = b4[i];
    y[4 * i] = __uint_as_float(u[4 * i]) + bb.x;
    y[4 * i + 1] = __uint_as_float(u[4 * i + 1]) + bb.y;
    y[4 * i + 2] = __uint_as_float(u[4 * i + 2]) + bb.z;
    y[4 * i + 3] = __uint_as_float(u[4 * i + 3]) + bb.w;
  }
}

// y in place: for q / k each pair rotated with token n's table entries.
__device__ __forceinline__ void rotate_pairs(const Params& p, int o_col, int n, bool rotate, float* r) {
  if (rotate) {
    const int pair0 = (o_col & 127) >> 1;       // first channel pair of the chunk within its head
    const float4* c4 = reinterpret_cast<const float4*>(p.cos + static_cast<size_t>(n) * 64 + pair0);
    const float4* s4 = reinterpret_cast<const float4*>(p.sin + static_cast<size_t>(n) * 64 + pair0);
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const float4 cc = __ldg(c4 + qd), ss = __ldg(s4 + qd);
      const float cs[4] = {cc.x, cc.y, cc.z, cc.w}, sn[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 8 * qd + 2 * e;
        const float a = r[i], bb = r[i + 1];
        r[i] = rot_f64(a, cs[e], bb, -sn[e]);
        r[i + 1] = rot_f64(a, sn[e], bb, cs[e]);
      }
    }
  }
}

// The epilogue of kHeads heads (128 accumulator columns each) for the 128
// token rows of this CTA starting at token n0, by two warp groups (warps 2-5
// and 6-9, one thread per row in each; warp w reads tensor-memory lanes
// 32 (w % 4) ...), each taking kHeads / 2 heads; sm supplies acc_full,
// block_max and the bias slice.  Per head: pass 1 loads y (+ bias), writes
// the optional bf16 y, rotates q / k pairs, takes the row amax and stores
// the final values back into the same tensor-memory columns; the block
// maxima of the two 64-token blocks come from a shuffle and shared-memory
// reduction over the group; pass 2 reloads the values and encodes them.
template <int kHeads, typename SmemT>
__device__ __forceinline__ void epilogue(SmemT& sm, const Params& p, uint32_t tmem, int n0, int o0, int b, int warp,
                                         int lane, const WaitCtx& wc) {
  constexpr int kGroupHeads = kHeads / 2;
  const int group = (warp - 2) >> 2;
  const int gt = ((warp - 2) & 3) * 32 + lane;     // thread within the group
  const int bar = kBarEpi + group;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const int n = n0 + row;
  const bool valid = n < p.N;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const int nb = (p.N + 63) / 64;
  // the group's bias columns into shared memory
  for (int i = gt; i < kGroupHeads * 128; i += kEpiThreads) {
    const int col = group * kGroupHeads * 128 + i;
    sm.bias[col] = p.bias != nullptr ? __ldg(p.bias + o0 + col) : 0.f;
  }
  named_bar_sync(bar, kEpiThreads);
  const bool ok = warp_wait(&sm.acc_full, 0, wc);
  tc_fence_after();
#pragma unroll 1
  for (int hh = 0; hh < kGroupHeads; ++hh) {
    const int head = group * kGroupHeads + hh;
    const int o_head = o0 + head * 128;            // first output feature of the head
    const int which = o_head / (p.H * 128);        // 0 q, 1 k, 2 v
    const int h = (o_head / 128) % p.H;
    const bool rotate = which < 2 && p.cos != nullptr && valid;
    const uint32_t tcol = tmem + lane_base + head * 128;
    uint8_t* const codes = which == 0 ? p.codes[0] : which == 1 ? p.codes[1] : p.codes[2];
    float* const scales = which == 0 ? p.scales[0] : which == 1 ? p.scales[1] : p.scales[2];
    __nv_bfloat16* const y16 = which == 0 ? p.y16[0] : which == 1 ? p.y16[1] : p.y16[2];
    // pass 1: y, the optional bf16 y, the rotation, the row amax; final values back to tensor memory
    float amax = 0.f;
    if (ok) {
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float r[32];
        load_y(tcol + q * 32, sm.bias + head * 128 + q * 32, r);
        if (valid && y16 != nullptr) {
          // unrotated y, rounded to bf16, in the attention layout
          uint4* dst = reinterpret_cast<uint4*>(y16 + ((static_cast<size_t>(b) * p.H + h) * p.N + n) * 128 + q * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pack_bf16x2_rn(r[8 * e], r[8 * e + 1]), pack_bf16x2_rn(r[8 * e + 2], r[8 * e + 3]),
                                pack_bf16x2_rn(r[8 * e + 4], r[8 * e + 5]), pack_bf16x2_rn(r[8 * e + 6], r[8 * e + 7]));
        }
        rotate_pairs(p, o_head + q * 32, n, rotate, r);
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(r[e]));
        }
        tmem_st32(tcol + q * 32, reinterpret_cast<const uint32_t*>(r));
      }
      tmem_st_wait();
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) sm.block_max[group * 4 + quarter] = amax;
    named_bar_sync(bar, kEpiThreads);
    const int blk = row >> 6;                      // 64-token block of the tile: quarters 0-1, 2-3
    const float bmax = fmaxf(sm.block_max[group * 4 + 2 * blk], sm.block_max[group * 4 + 2 * blk + 1]);
    named_bar_sync(bar, kEpiThreads);              // block_max is reused by the next head
    const float scale = bmax == 0.f ? 1.0f : __fdiv_rn(bmax, 448.0f);
    if ((row & 63) == 0 && valid) scales[(static_cast<size_t>(b) * p.H + h) * nb + (n0 >> 6) + blk] = scale;
    if (!ok) continue;
    // pass 2: the codes of r / scale (the reciprocal decides when it can);
    // every lane takes part in the warp-collective loads, valid rows store
    const bool via_reciprocal = scale >= 1.17549435e-38f && scale <= 8.50705917e+37f;
    const float rs = __frcp_rn(scale);
    uint8_t* out = codes + ((static_cast<size_t>(b) * p.H + h) * p.N + n) * 128;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      uint32_t u[32];
      tmem_ld32(tcol + q * 32, u);
      tmem_ld_wait(u);
      const float* r = reinterpret_cast<const float*>(u);
      uint32_t word[8];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (!via_reciprocal || !e4m3x8_of_quotients(r + 8 * g, rs, word[2 * g], word[2 * g + 1]))
          e4m3x8_by_division(r + 8 * g, scale, word[2 * g], word[2 * g + 1]);
      }
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + q * 32);
        dst[0] = make_uint4(word[0], word[1], word[2], word[3]);
        dst[1] = make_uint4(word[4], word[5], word[6], word[7]);
      }
    }
  }
}

// ---------------------------------------------------------------- CTA pairs
// A cluster of two CTAs computes 256 tokens (128 per CTA) x kHeads heads
// (128 output features each) with pair MMAs (M = 256, N = 256, one per 256
// features and 16 input channels, into tensor-memory columns 0-255, 256-511).
// Each CTA loads its own 128 token rows of x and, for each 256-feature MMA,
// its half (128 weight rows); the pair MMA reads both CTAs' halves.  kHeads =
// 4 (512 features) loads 48 KB per 64 channels per CTA into a 4-stage ring and
// holds all 512 tensor-memory columns: one CTA per SM, and the epilogue of a
// tile does not overlap any MMA.  kHeads = 2 loads 32 KB per 64 channels into
// a 3-stage ring and holds 256 columns, so two CTAs share an SM and one's
// epilogue runs while the other's MMAs do.  The epilogue is the one above.
template <int kHeads>
struct PairCfg {
  static constexpr int kBN = kHeads * 128;                 // output features per tile
  static constexpr int kMmas = kBN / 256;                  // N = 256 pair MMAs per 16 channels
  static constexpr int kStages = kHeads == 4 ? 4 : 3;
  static constexpr int kMinBlocks = kHeads == 4 ? 1 : 2;   // CTAs per SM
  static constexpr int kBHalf = 128 * kBK * 2;             // 16 KB: 128 weight rows of one MMA
  static constexpr int kStageBytes = kABytes + kMmas * kBHalf;
};

template <int kHeads>
struct __align__(1024) PairSmem {
  using Cfg = PairCfg<kHeads>;
  uint8_t a[Cfg::kStages][kABytes];
  uint8_t b[Cfg::kStages][Cfg::kMmas][Cfg::kBHalf];
  uint64_t full[Cfg::kStages], empty[Cfg::kStages];   // full: the even CTA's counts both CTAs' bytes
  uint64_t acc_full;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
  float block_max[8];
  alignas(16) float bias[Cfg::kBN];
};

__device__ __forceinline__ uint32_t cl_addr(const void* p, uint32_t rank) { return mapa_shared(smem_u32(p), rank); }

template <int kHeads>
__device__ __forceinline__ void pair_producer(PairSmem<kHeads>& sm, const Params& p, const CUtensorMap* tm_x,
                                              const CUtensorMap* tm_w, int n0, int o0, int b, uint32_t rank,
                                              const WaitCtx& wc) {
  using Cfg = PairCfg<kHeads>;
  tma_prefetch_desc(tm_x);
  tma_prefetch_desc(tm_w);
  int issued = 0;
  for (int k = 0; k < p.k_steps; ++k) {
    const int s = k % Cfg::kStages;
    const uint32_t ph = (k / Cfg::kStages) & 1;
    if (!mbar_wait(&sm.empty[s], ph ^ 1, wc)) break;
    if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 2 * Cfg::kStageBytes);
    const uint32_t bar = cl_addr(&sm.full[s], 0);
    tma_load_3d_pair(sm.a[s], tm_x, bar, k * kBK, n0, b);
    for (int m = 0; m < Cfg::kMmas; ++m)
      tma_load_3d_pair(sm.b[s][m], tm_w, bar, k * kBK, o0 + 256 * m + 128 * static_cast<int>(rank), 0);
    issued = k + 1;
  }
  if (*wc.abort) {
    // let the copies already issued land before the pair exits: the even CTA
    // counts both CTAs' bytes; the odd CTA waits out a few microseconds
    if (rank == 0) {
      for (int k = (issued > Cfg::kStages ? issued - Cfg::kStages : 0); k < issued; ++k)
        mbar_wait_drain(&sm.full[k % Cfg::kStages], (k / Cfg::kStages) & 1, wc);
    } else {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 20000) {
      }
    }
  }
}

// Even CTA only: completions are signalled to the barrier of the same name in
// both CTAs.
template <int kHeads>
__device__ __forceinline__ void pair_mma_issuer(PairSmem<kHeads>& sm, const Params& p, uint32_t tmem,
                                                const WaitCtx& wc) {
  using Cfg = PairCfg<kHeads>;
  constexpr uint32_t idesc = instr_desc(1, 1, 256, 256, 0, 0);    // bf16 x bf16 -> fp32, both K-major
  const uint64_t a0 = smem_desc_sw128(smem_u32(sm.a[0]), 16, 1024);
  const uint64_t b0 = smem_desc_sw128(smem_u32(sm.b[0][0]), 16, 1024);
  bool ok = true;
  for (int k = 0; k < p.k_steps; ++k) {
    const int s = k % Cfg::kStages;
    if (!(ok = mbar_wait(&sm.full[s], (k / Cfg::kStages) & 1, wc))) break;
    tc_fence_after();
    const uint64_t ad = a0 + static_cast<uint32_t>(s) * (kABytes >> 4);
    const uint64_t bd = b0 + static_cast<uint32_t>(s) * ((Cfg::kMmas * Cfg::kBHalf) >> 4);
#pragma unroll
    for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
      for (int m = 0; m < Cfg::kMmas; ++m)
        mma_ss_pair(tmem + 256 * m, ad + kk * 2, bd + m * (Cfg::kBHalf >> 4) + kk * 2, idesc,
                    (k > 0 || kk > 0) ? 1u : 0u);
    }
    tc_commit_pair(cl_addr(&sm.empty[s], 0));
    tc_commit_pair(cl_addr(&sm.empty[s], 1));
  }
  if (ok) {
    tc_commit_pair(cl_addr(&sm.acc_full, 0));
    tc_commit_pair(cl_addr(&sm.acc_full, 1));
  }
  // every MMA issued above has completed once this arrives
  tc_commit_pair(cl_addr(&sm.mma_drain, 0));
  mbar_wait_drain(&sm.mma_drain, 0, wc);
}

template <int kHeads>
__global__ void __launch_bounds__(kThreads, PairCfg<kHeads>::kMinBlocks)
    qkv_proj_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const Params p) {
  using Cfg = PairCfg<kHeads>;
  extern __shared__ uint8_t smem_raw[];
  PairSmem<kHeads>& sm =
      *reinterpret_cast<PairSmem<kHeads>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  // clusters are two CTAs along x: blockIdx.x = 2 x (feature tile) + rank, so that the
  // feature tiles of one token tile run next to each other and the weight stays in L2
  const int n0 = blockIdx.y * 2 * kBM + kBM * static_cast<int>(rank);   // this CTA's first token
  const int o0 = (blockIdx.x >> 1) * Cfg::kBN;
  const int b = blockIdx.z;
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.mma_drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, Cfg::kBN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();          // both CTAs' barriers initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort, p.status, cl_addr(&sm.abort, rank ^ 1u)};
  if (warp == 0) {
    if (lane == 0) pair_producer<kHeads>(sm, p, &tm_x, &tm_w, n0, o0, b, rank, wc);
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) pair_mma_issuer<kHeads>(sm, p, tmem, wc);
  } else {
    epilogue<kHeads>(sm, p, tmem, n0, o0, b, warp, lane, wc);
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();          // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, Cfg::kBN);
}

bool make_map(CUtensorMap* map, const void* base, int inner, int rows, int planes, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2,
                                 static_cast<cuuint64_t>(inner) * rows * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Heads per CTA-pair tile: 2 (two CTAs per SM, epilogue overlapped with the
// other CTA's MMAs) or 4 (one CTA per SM; H a multiple of 4).  Measured at
// 2048²: 0.782 against 0.797 ms, the codes bit-identical.
constexpr int kPairHeads = 2;

template <int kHeads>
int launch_pair(const CUtensorMap& mx, const CUtensorMap& mw, const Params& p, int B, cudaStream_t s) {
  using Cfg = PairCfg<kHeads>;
  const size_t smem = sizeof(PairSmem<kHeads>) + 1024;
  static thread_local int configured_device = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -4;
  if (configured_device != dev) {
    if (cudaFuncSetAttribute(qkv_proj_pair_kernel<kHeads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(qkv_proj_pair_kernel<kHeads>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             static_cast<int>(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return -4;
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (3 * p.H * 128 / Cfg::kBN), (p.N + 2 * kBM - 1) / (2 * kBM), B);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qkv_proj_pair_kernel<kHeads>, mx, mw, p) == cudaSuccess ? 0 : -4;
}

int launch_qkv_proj_fp8(const QkvProjArgs& a, cudaStream_t s) {
  // the tile's 128 * kPairHeads features must divide the 3 H heads' 3 H 128
  if ((3 * a.H) % kPairHeads != 0) return -2;
  CUtensorMap mx, mw;
  if (!make_map(&mx, a.x, a.C, a.N, a.B, kBM) || !make_map(&mw, a.w, a.C, 3 * a.H * 128, 1, 128)) return -4;
  Params p;
  p.bias = a.bias;
  p.cos = a.cos;
  p.sin = a.sin;
  for (int i = 0; i < 3; ++i) {
    p.codes[i] = a.codes[i];
    p.scales[i] = a.scales[i];
    p.y16[i] = static_cast<__nv_bfloat16*>(a.y16[i]);
  }
  p.status = device_status_word();
  if (p.status == nullptr) return -4;
  p.N = a.N;
  p.C = a.C;
  p.H = a.H;
  p.k_steps = (a.C + kBK - 1) / kBK;
  return launch_pair<kPairHeads>(mx, mw, p, a.B, s);
}

}  // namespace dit
