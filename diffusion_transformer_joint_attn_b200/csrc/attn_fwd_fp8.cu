// Joint text+image attention forward on FP8 E4M3 operands (sm_100a).
//
// Same CTA-pair pipeline as the BF16 kernel: a cluster of two CTAs owns four
// 128-row query tiles of one (b, h) as two 256-row slots, and streams every
// 128-key tile past them with an online softmax.  Differences:
//   * Q and K arrive as E4M3 codes with one fp32 scale per 64 tokens (from
//     dit_attn_quantize_fp8, rotary embedding already applied): S = Q K^T is
//     a kind::f8f6f4 pair MMA on the codes; the softmax multiplies each half
//     of a key tile by q_scale(row block) * k_scale(key block), folded into
//     its exponent's fused multiply-add.
//   * V arrives as E4M3 codes + scales; warps 2-3 turn each V half tile into
//     fp16 values code * scale (fp32 product, rounded once) in the
//     128B-swizzled layout the P V MMA reads, so P V keeps fp16 precision.
//
// Roles, by warp:   0 TMA producer | 1 MMA issuer (even CTA) | 2-3 V
// dequantisation | 4-7, 8-11 softmax of slot 0 / 1.  Twelve warps leave 168
// registers per thread (65536 / 384), enough for a softmax row without
// setmaxnreg, whose mere presence in a kernel slows its pair-MMA issue.
#include "attn_common.cuh"
#include "launch.h"

namespace dit {
namespace {

using attn::cl;
using attn::commit_both;
using attn::kHeadDim;
using attn::kTile;
using attn::pack_f16;
using attn::Pair;

constexpr int kStages = 4;
constexpr int kQ8Bytes = kTile * kHeadDim;         // 16 KB: 128 rows x 128 codes
constexpr int kK8HalfBytes = 64 * kHeadDim;        // 8 KB: 64 keys x 128 codes
constexpr int kV8HalfBytes = kTile * 64;           // 8 KB: 128 keys x 64 codes, unswizzled
constexpr int kVHalfBytes = kTile * 64 * 2;        // 16 KB: 128 keys x 64 fp16, 128B swizzle
constexpr int kThreads = 384;
constexpr int kCvtWarps = 2;                       // warps 2-3
constexpr int kCvtThreads = kCvtWarps * 32;

struct __align__(1024) Smem {
  uint8_t q[2][kQ8Bytes];
  uint8_t k[kStages][kK8HalfBytes];
  uint8_t v8[kStages][kV8HalfBytes];
  uint8_t v[kStages][kVHalfBytes];
  uint64_t q_full;                                   // even CTA: both CTAs' Q codes
  uint64_t k_full[kStages];
  uint64_t kv_empty[kStages];                        // stage s free again: P V of its tile has completed
  uint64_t v8_full[kStages], v8_empty[kStages];      // local staging ring
  uint64_t v_ready[kStages];
  uint64_t s_full[2], p_ready[2], o_final[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  void* out;
  float* lse;
  int* status;
  const float* q_scale;   // [B*H][n_blocks]
  const float* k_scale;
  const float* v_scale;
  int N;
  int n_kv;
  int n_blocks;
  int clusters;
  int out_f32;
  float scale_log2;
};

__device__ __forceinline__ void producer_role(Smem& sm, const Params& p, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k, const CUtensorMap* tm_v, const Pair& pr,
                                              const WaitCtx& wc) {
  tma_prefetch_desc(tm_q);
  tma_prefetch_desc(tm_k);
  tma_prefetch_desc(tm_v);
  const bool leader = pr.rank == 0;
  if (leader) mbar_arrive_expect_tx(&sm.q_full, 4 * kQ8Bytes);
  for (int t = 0; t < 2; ++t) tma_load_3d_pair(sm.q[t], tm_q, cl(&sm.q_full, 0), 0, pr.row0[t], pr.bh);
  int issued = 0;
  for (int j = 0; j < p.n_kv; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (j / kStages) & 1;
    const int key0 = j * kTile;
    if (!mbar_wait(&sm.kv_empty[s], ph ^ 1, wc)) break;
    if (leader) mbar_arrive_expect_tx(&sm.k_full[s], 2 * kK8HalfBytes);
    tma_load_3d_pair(sm.k[s], tm_k, cl(&sm.k_full[s], 0), 0, key0 + 64 * static_cast<int>(pr.rank), pr.bh);
    if (!mbar_wait(&sm.v8_empty[s], ph ^ 1, wc)) {
      issued = 2 * j + 1;
      break;
    }
    mbar_arrive_expect_tx(&sm.v8_full[s], kV8HalfBytes);
    tma_load_3d(sm.v8[s], tm_v, &sm.v8_full[s], 64 * static_cast<int>(pr.rank), key0, pr.bh);
    issued = 2 * j + 2;
  }
  if (*wc.abort) {
    // Let the copies already issued land before the pair exits (see the BF16
    // kernel); the odd CTA waits out a few microseconds for its pair loads.
    for (int i = (issued > 2 * kStages ? issued - 2 * kStages : 0); i < issued; ++i) {
      const int j = i / 2, s = j % kStages;
      const uint32_t ph = (j / kStages) & 1;
      if (i & 1)
        mbar_wait_drain(&sm.v8_full[s], ph, wc);
      else if (leader)
        mbar_wait_drain(&sm.k_full[s], ph, wc);
    }
    if (leader) {
      mbar_wait_drain(&sm.q_full, 0, wc);
    } else {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 20000) {
      }
    }
  }
}

__device__ __forceinline__ void mma_role(Smem& sm, const Params& p, uint32_t tmem, const WaitCtx& wc) {
  constexpr uint32_t idesc_qk = instr_desc(0, 0, 256, 128, 0, 0);   // e4m3 x e4m3, both K-major
  constexpr uint32_t idesc_pv = instr_desc(0, 0, 256, 128, 0, 1);   // f16 x f16, V MN-major
  const uint64_t q_desc0 = smem_desc_sw128(smem_u32(sm.q[0]), 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(smem_u32(sm.k[0]), 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(smem_u32(sm.v[0]), kVHalfBytes, 1024);
  bool ok = mbar_wait(&sm.q_full, 0, wc);
  tc_fence_after();
  for (int j = 0; ok && j <= p.n_kv; ++j) {
    const int s = j % kStages;
    const int sp = (j + kStages - 1) % kStages;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t tS = tmem + t * 128;
      const uint32_t tO = tmem + 256 + t * 128;
      if (j > 0) {
        if (!(ok = mbar_wait(&sm.p_ready[t], (j - 1) & 1, wc))) break;
        if (t == 0 && !(ok = mbar_wait(&sm.v_ready[sp], ((j - 1) / kStages) & 1, wc))) break;
        tc_fence_after();
        const uint64_t vd = v_desc0 + static_cast<uint32_t>(sp) * (kVHalfBytes >> 4);
        mma_ts_pair(tO, tS, vd, idesc_pv, j > 1 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) mma_ts_pair(tO, tS + kk * 8, vd + kk * (2048 >> 4), idesc_pv, 1u);
        if (j == p.n_kv) commit_both(&sm.o_final[t]);
      }
      if (j < p.n_kv) {
        if (t == 0) {
          if (!(ok = mbar_wait(&sm.k_full[s], (j / kStages) & 1, wc))) break;
          tc_fence_after();
        }
        const uint64_t qd = q_desc0 + t * (kQ8Bytes >> 4);
        const uint64_t kd = k_desc0 + static_cast<uint32_t>(s) * (kK8HalfBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_ss_pair_f8(tS, qd + kk * 2, kd + kk * 2, idesc_qk, kk > 0 ? 1u : 0u);
        commit_both(&sm.s_full[t]);
      }
    }
    if (!ok) break;
    // one release per stage: the commit tracks Q K_{j-1}^T and P V_{j-1}
    if (j > 0) commit_both(&sm.kv_empty[sp]);
  }
  tc_commit_pair(cl(&sm.mma_drain, 0));
  mbar_wait_drain(&sm.mma_drain, 0, wc);
}

// Two E4M3 codes (low byte first) -> fp32 pair (exact).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t two) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(two));
  return __half22float2(*reinterpret_cast<__half2*>(&h));
}

// Warps 2-3: V_j codes -> fp16 values code * scale in the swizzled operand
// layout (row = key, 8-channel chunk c at chunk c ^ (key & 7)).
__device__ __forceinline__ void dequant_v_role(Smem& sm, const Params& p, const Pair& pr, int warp, int lane,
                                               const WaitCtx& wc) {
  const int pt = (warp - 2) * 32 + lane;
  const float* vscale = p.v_scale + static_cast<size_t>(pr.bh) * p.n_blocks;
  for (int j = 0; j < p.n_kv; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (j / kStages) & 1;
    if (!warp_wait(&sm.v8_full[s], ph, wc)) break;
    if (!warp_wait(&sm.kv_empty[s], ph ^ 1, wc)) break;
    const int blk0 = 2 * j;
    const float vs0 = __ldg(vscale + blk0);
    const float vs1 = blk0 + 1 < p.n_blocks ? __ldg(vscale + blk0 + 1) : vs0;
    for (int c = pt; c < kTile * 8; c += kCvtThreads) {
      const int r = c >> 3, c8 = c & 7;
      const uint2 w = *reinterpret_cast<const uint2*>(sm.v8[s] + r * 64 + c8 * 8);
      const float2 vs = r < 64 ? make_float2(vs0, vs0) : make_float2(vs1, vs1);
      const float2 a = __fmul2_rn(e4m3x2_to_f32x2(static_cast<uint16_t>(w.x)), vs);
      const float2 b = __fmul2_rn(e4m3x2_to_f32x2(static_cast<uint16_t>(w.x >> 16)), vs);
      const float2 d = __fmul2_rn(e4m3x2_to_f32x2(static_cast<uint16_t>(w.y)), vs);
      const float2 e = __fmul2_rn(e4m3x2_to_f32x2(static_cast<uint16_t>(w.y >> 16)), vs);
      *reinterpret_cast<uint4*>(sm.v[s] + r * 128 + ((c8 ^ (r & 7)) << 4)) =
          make_uint4(pack_f16(a.x, a.y), pack_f16(b.x, b.y), pack_f16(d.x, d.y), pack_f16(e.x, e.y));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&sm.v8_empty[s]);
      mbar_arrive_cluster(cl(&sm.v_ready[s], 0));   // release at cluster scope: the peer's MMA reads sm.v
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  Pair pr;
  pr.rank = cluster_ctarank();
  pr.peer = pr.rank ^ 1u;
  const int cluster = blockIdx.x >> 1;
  pr.bh = cluster / p.clusters;
  const int q0 = (cluster % p.clusters) * 4 * kTile;
  pr.row0[0] = q0 + kTile * static_cast<int>(pr.rank);
  pr.row0[1] = q0 + 2 * kTile + kTile * static_cast<int>(pr.rank);

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
      mbar_init(&sm.v8_full[s], 1);
      mbar_init(&sm.v8_empty[s], kCvtWarps);
      mbar_init(&sm.v_ready[s], 2 * kCvtWarps);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_ready[t], 8);
      mbar_init(&sm.o_final[t], 1);
    }
    mbar_init(&sm.mma_drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort, p.status, cl(&sm.abort, pr.peer)};

  const int wg = warp >> 2;
  if (wg == 1 || wg == 2) {
    const size_t base = static_cast<size_t>(pr.bh) * p.n_blocks;
    attn::SoftmaxIo io{sm.s_full, sm.p_ready, sm.o_final, p.out, p.lse, p.N, p.N, p.n_kv, p.out_f32,
                       p.scale_log2, p.q_scale + base, p.k_scale + base, p.n_blocks, nullptr, p.n_kv};
    attn::softmax_slot<true>(io, tmem, pr, warp, lane, wc);
  } else {
    if (warp == 0) {
      if (lane == 0) producer_role(sm, p, &tm_q, &tm_k, &tm_v, pr, wc);
    } else if (warp == 1) {
      if (lane == 0 && pr.rank == 0) mma_role(sm, p, tmem, wc);
    } else {
      dequant_v_role(sm, p, pr, warp, lane, wc);
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

bool make_map_u8(CUtensorMap* map, const void* base, int BH, int N, int box_x, int box_rows, bool swizzle) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(N) * kHeadDim};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int launch_attn_fwd_fp8(const AttnFwdFp8Args& a, cudaStream_t s) {
  const int BH = a.B * a.H;
  CUtensorMap mq, mk, mv;
  if (!make_map_u8(&mq, a.q8, BH, a.N, 128, kTile, true) || !make_map_u8(&mk, a.k8, BH, a.N, 128, 64, true) ||
      !make_map_u8(&mv, a.v8, BH, a.N, 64, kTile, false))
    return -4;
  Params p;
  p.out = a.out;
  p.lse = a.lse;
  p.status = device_status_word();
  if (p.status == nullptr) return -4;
  p.q_scale = a.q_scale;
  p.k_scale = a.k_scale;
  p.v_scale = a.v_scale;
  p.N = a.N;
  p.n_kv = (a.N + kTile - 1) / kTile;
  p.n_blocks = (a.N + 63) / 64;
  p.clusters = (a.N + 4 * kTile - 1) / (4 * kTile);
  p.out_f32 = a.out_f32 ? 1 : 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kHeadDim));
  const long long grid = 2LL * BH * p.clusters;
  if (grid > 0x7FFFFFFFLL) return -1;
  const size_t smem = sizeof(Smem) + 1024;
  static thread_local int configured_device = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -4;
  if (configured_device != dev) {
    if (cudaFuncSetAttribute(attn_fwd_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -4;
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
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
  return cudaLaunchKernelEx(&cfg, attn_fwd_fp8_kernel, mq, mk, mv, p) == cudaSuccess ? 0 : -4;
}

}  // namespace dit
