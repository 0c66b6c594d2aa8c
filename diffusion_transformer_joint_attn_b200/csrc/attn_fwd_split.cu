// Joint attention forward with a compensated q~ k~^T (sm_100a): the "split"
// form, for inputs whose logits are large enough that one bf16 rounding of
// the rotated q and k moves the result (activation-outlier channels x16 give
// logits with a standard deviation of ~45, where a bf16 operand error of
// 2^-9 shifts a logit by ~0.1).
//
// Each rotated operand r (fp32, rope_split.cuh) is carried by two fp16 terms
// hi + lo, and S = Q K^T is accumulated in fp32 tensor memory from three
// products per 128-key tile:
//     S = Q_hi K_lo^T + Q_lo K_hi^T + Q_hi K_hi^T
// (the small cross terms first; lo * lo, ~2^-22 relative, is left out).  The
// rest is the pipeline of the BF16 kernel (attn_fwd.cu): a CTA pair owns four
// 128-row query tiles of one (b, h) as two 256-row slots, the even CTA issues
// pair MMAs (M = 256) over each CTA's half of every K / V tile, the online
// softmax and epilogue are the shared ones of attn_common.cuh, P and V enter
// P V as fp16.
//
// Differences forced by the extra operands: Q_hi and Q_lo of both slots take
// 128 KB of shared memory, so the K and V rings have two stages, with K and V
// stages released separately (K as soon as both slots' S of the tile have
// completed) so that each load has a whole tile of lead.  K comes prepared
// by dit_attn_prepare_kv_split (rotated and split once per call); Q is
// rotated and split in the prologue by warps 2-11.
//
// Roles, by warp: 0 TMA producer | 1 MMA issuer (even CTA) | 2-11 Q rotation
// and split (prologue) | 4-7, 8-11 softmax of slot 0 / 1.
#include "attn_common.cuh"
#include "launch.h"
#include "rope_split.cuh"

namespace dit {
namespace {

using attn::cl;
using attn::commit_both;
using attn::kHeadDim;
using attn::kTile;
using attn::Pair;

constexpr int kStages = 2;
constexpr int kQTileBytes = kTile * kHeadDim * 2;  // 32 KB: 128 rows x 128 channels (fp16)
constexpr int kQBoxBytes = kTile * 64 * 2;         // 16 KB: 128 rows x 64 channels
constexpr int kKHalfBytes = 64 * kHeadDim * 2;     // 16 KB: 64 keys x 128 channels
constexpr int kKBoxBytes = 64 * 64 * 2;            // 8 KB: 64 keys x 64 channels
constexpr int kVHalfBytes = kTile * 64 * 2;        // 16 KB: 128 keys x 64 channels
constexpr int kThreads = 384;
constexpr int kPrologueThreads = kThreads - 64;    // warps 2-11
constexpr int kBarQSplit = 1;                      // named barrier of the Q prologue

struct __align__(1024) Smem {
  uint8_t q_hi[2][kQTileBytes];   // the TMA lands the bf16 Q here; the prologue overwrites it with hi
  uint8_t q_lo[2][kQTileBytes];
  uint8_t k_hi[kStages][kKHalfBytes];
  uint8_t k_lo[kStages][kKHalfBytes];
  uint8_t v[kStages][kVHalfBytes];
  uint64_t q_full;
  uint64_t q_ready;                                  // even CTA: one arrive per CTA
  uint64_t k_full[kStages], k_empty[kStages];        // k_empty: both slots' S of the stage's tile completed
  uint64_t v_full[kStages], v_empty[kStages];        // v_empty: both slots' P V of the stage's tile completed
  uint64_t s_full[2], p_ready[2], o_final[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory of the split kernel");

struct Params {
  const float* cos;   // [N][64] or nullptr
  const float* sin;
  void* out;
  float* lse;
  int* status;
  int BH;
  int N;              // query rows per (b, h)
  int N_kv;           // keys per (b, h)
  int n_kv;
  int clusters;
  int out_f32;
  float scale_log2;
};

// Q tile chunk c (0..2047): byte offset in the 128B-swizzled layout of two
// 128-row x 64-channel boxes, its row and first channel.
__device__ __forceinline__ void q_chunk(int c, int& byte_off, int& row, int& col0) {
  const int box = c >> 10;
  row = (c >> 3) & 127;
  const int phys = c & 7;
  byte_off = box * kQBoxBytes + row * 128 + phys * 16;
  col0 = box * 64 + ((phys ^ (row & 7)) << 3);
}

__device__ __forceinline__ void producer_role(Smem& sm, const Params& p, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k, const CUtensorMap* tm_v, const Pair& pr,
                                              const WaitCtx& wc) {
  tma_prefetch_desc(tm_q);
  tma_prefetch_desc(tm_k);
  tma_prefetch_desc(tm_v);
  mbar_arrive_expect_tx(&sm.q_full, 2 * kQTileBytes);
  for (int t = 0; t < 2; ++t)
    for (int b = 0; b < 2; ++b)
      tma_load_3d(sm.q_hi[t] + b * kQBoxBytes, tm_q, &sm.q_full, b * 64, pr.row0[t], pr.bh);
  const bool leader = pr.rank == 0;
  const int key_half = 64 * static_cast<int>(pr.rank);
  int issued = 0;
  for (int j = 0; j < p.n_kv; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (j / kStages) & 1;
    const int key0 = j * kTile;
    if (!mbar_wait(&sm.k_empty[s], ph ^ 1, wc)) break;
    if (leader) mbar_arrive_expect_tx(&sm.k_full[s], 4 * kKHalfBytes);
    const uint32_t kbar = cl(&sm.k_full[s], 0);
    for (int b = 0; b < 2; ++b) {
      tma_load_3d_pair(sm.k_hi[s] + b * kKBoxBytes, tm_k, kbar, b * 64, key0 + key_half, pr.bh);
      tma_load_3d_pair(sm.k_lo[s] + b * kKBoxBytes, tm_k, kbar, b * 64, key0 + key_half, p.BH + pr.bh);
    }
    issued = 2 * j + 1;
    if (!mbar_wait(&sm.v_empty[s], ph ^ 1, wc)) break;
    if (leader) mbar_arrive_expect_tx(&sm.v_full[s], 2 * kVHalfBytes);
    tma_load_3d_pair(sm.v[s], tm_v, cl(&sm.v_full[s], 0), key_half, key0, pr.bh);
    issued = 2 * j + 2;
  }
  if (*wc.abort) {
    // Let the copies already issued land before the pair exits: the even CTA
    // counts the bytes of both CTAs' pair loads; the odd CTA waits out a few
    // microseconds instead.
    mbar_wait_drain(&sm.q_full, 0, wc);
    if (leader) {
      for (int i = (issued > 2 * kStages ? issued - 2 * kStages : 0); i < issued; ++i) {
        const int j = i / 2, s = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        mbar_wait_drain((i & 1) ? &sm.v_full[s] : &sm.k_full[s], ph, wc);
      }
    } else {
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < 20000) {
      }
    }
  }
}

// Even CTA only.
__device__ __forceinline__ void mma_role(Smem& sm, const Params& p, uint32_t tmem, const WaitCtx& wc) {
  constexpr uint32_t idesc_qk = instr_desc(0, 0, 256, 128, 0, 0);   // f16 x f16, both K-major
  constexpr uint32_t idesc_pv = instr_desc(0, 0, 256, 128, 0, 1);   // f16 x f16, V MN-major
  const uint64_t qh_desc0 = smem_desc_sw128(smem_u32(sm.q_hi[0]), 16, 1024);
  const uint64_t ql_desc0 = smem_desc_sw128(smem_u32(sm.q_lo[0]), 16, 1024);
  const uint64_t kh_desc0 = smem_desc_sw128(smem_u32(sm.k_hi[0]), 16, 1024);
  const uint64_t kl_desc0 = smem_desc_sw128(smem_u32(sm.k_lo[0]), 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(smem_u32(sm.v[0]), kVHalfBytes, 1024);
  bool ok = mbar_wait(&sm.q_ready, 0, wc);
  tc_fence_after();
  for (int j = 0; ok && j <= p.n_kv; ++j) {
    const int s = j % kStages;
    const int sp = (j + kStages - 1) % kStages;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t tS = tmem + t * 128;
      const uint32_t tO = tmem + 256 + t * 128;
      if (j > 0) {
        // O_t += P_t V_{j-1}
        if (!(ok = mbar_wait(&sm.p_ready[t], (j - 1) & 1, wc))) break;
        if (t == 0 && !(ok = mbar_wait(&sm.v_full[sp], ((j - 1) / kStages) & 1, wc))) break;
        tc_fence_after();
        const uint64_t vd = v_desc0 + static_cast<uint32_t>(sp) * (kVHalfBytes >> 4);
        mma_ts_pair(tO, tS, vd, idesc_pv, j > 1 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) mma_ts_pair(tO, tS + kk * 8, vd + kk * (2048 >> 4), idesc_pv, 1u);
        if (j == p.n_kv) commit_both(&sm.o_final[t]);
      }
      if (j < p.n_kv) {
        // S_t = Q_t K_j^T from the three hi / lo products
        if (t == 0) {
          if (!(ok = mbar_wait(&sm.k_full[s], (j / kStages) & 1, wc))) break;
          tc_fence_after();
        }
        const uint64_t qh = qh_desc0 + t * (kQTileBytes >> 4);
        const uint64_t ql = ql_desc0 + t * (kQTileBytes >> 4);
        const uint64_t kh = kh_desc0 + static_cast<uint32_t>(s) * (kKHalfBytes >> 4);
        const uint64_t kl = kl_desc0 + static_cast<uint32_t>(s) * (kKHalfBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = ((kk >> 2) * kQBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t boff = ((kk >> 2) * kKBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss_pair(tS, qh + aoff, kl + boff, idesc_qk, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = ((kk >> 2) * kQBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t boff = ((kk >> 2) * kKBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss_pair(tS, ql + aoff, kh + boff, idesc_qk, 1u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = ((kk >> 2) * kQBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t boff = ((kk >> 2) * kKBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss_pair(tS, qh + aoff, kh + boff, idesc_qk, 1u);
        }
        commit_both(&sm.s_full[t]);
        // both slots' S of tile j are issued: K_j's stage is free once they complete
        if (t == 1) commit_both(&sm.k_empty[s]);
      }
    }
    if (!ok) break;
    // both slots' P V_{j-1} are issued: V_{j-1}'s stage is free once they complete
    if (j > 0) commit_both(&sm.v_empty[sp]);
  }
  // every MMA issued above has completed once this arrives
  tc_commit_pair(cl(&sm.mma_drain, 0));
  mbar_wait_drain(&sm.mma_drain, 0, wc);
}

// Warps 2-11: rotate the CTA's two bf16 Q tiles and split them into the
// fp16 hi (in place) and lo tiles, then one arrive on the even CTA's q_ready.
// Rows past N were zero-filled by the TMA load; zero splits into zeros.
__device__ __forceinline__ void split_q(Smem& sm, const Params& p, const Pair& pr, int warp, int lane,
                                        const WaitCtx& wc) {
  const int qt = (warp - 2) * 32 + lane;
  const bool ok = warp_wait(&sm.q_full, 0, wc);
  if (ok) {
    for (int c = qt; c < 2 * (kQTileBytes / 16); c += kPrologueThreads) {
      const int t = c / (kQTileBytes / 16);
      int off, row, col0;
      q_chunk(c % (kQTileBytes / 16), off, row, col0);
      const int n = pr.row0[t] + row;
      const bool rotate = p.cos != nullptr && n < p.N;
      const uint4 x = *reinterpret_cast<const uint4*>(sm.q_hi[t] + off);
      float4 cs = make_float4(1.f, 1.f, 1.f, 1.f), sn = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rotate) {
        const int j0 = n * (kHeadDim / 2) + (col0 >> 1);
        cs = __ldg(reinterpret_cast<const float4*>(p.cos + j0));
        sn = __ldg(reinterpret_cast<const float4*>(p.sin + j0));
      }
      uint4 hi, lo;
      split_pair_f16(rotate_pair_f32(x.x, cs.x, sn.x, rotate), hi.x, lo.x);
      split_pair_f16(rotate_pair_f32(x.y, cs.y, sn.y, rotate), hi.y, lo.y);
      split_pair_f16(rotate_pair_f32(x.z, cs.z, sn.z, rotate), hi.z, lo.z);
      split_pair_f16(rotate_pair_f32(x.w, cs.w, sn.w, rotate), hi.w, lo.w);
      *reinterpret_cast<uint4*>(sm.q_hi[t] + off) = hi;
      *reinterpret_cast<uint4*>(sm.q_lo[t] + off) = lo;
    }
  }
  fence_proxy_async_smem();
  named_bar_sync(kBarQSplit, kPrologueThreads);
  if (ok && qt == 0) mbar_arrive_cluster(cl(&sm.q_ready, 0));
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
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
    mbar_init(&sm.q_ready, 2);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
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
  cluster_sync();          // both CTAs' barriers initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort, p.status, cl(&sm.abort, pr.peer)};

  const int wg = warp >> 2;
  if (wg == 1 || wg == 2) {
    split_q(sm, p, pr, warp, lane, wc);
    attn::SoftmaxIo io{sm.s_full, sm.p_ready, sm.o_final, p.out, p.lse, p.N, p.N_kv, p.n_kv, p.out_f32,
                       p.scale_log2, nullptr, nullptr, 0, nullptr, p.n_kv};
    attn::softmax_slot<false, false>(io, tmem, pr, warp, lane, wc);
  } else if (warp == 0) {
    if (lane == 0) producer_role(sm, p, &tm_q, &tm_k, &tm_v, pr, wc);
  } else if (warp == 1) {
    if (lane == 0 && pr.rank == 0) mma_role(sm, p, tmem, wc);
  } else {
    split_q(sm, p, pr, warp, lane, wc);
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();          // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

// 3-D map (D, N, planes) of 16-bit elements, 64-channel x box_rows boxes with
// the 128-byte swizzle.
bool make_map16(CUtensorMap* map, const void* base, int planes, int N, CUtensorMapDataType type, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                 static_cast<cuuint64_t>(N) * kHeadDim * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const CUresult r = enc(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int launch_attn_fwd_split(const AttnFwdSplitArgs& a, cudaStream_t s) {
  const int BH = a.B * a.H;
  if (BH > 0x3FFFFFFF) return -1;
  const int N_kv = a.N_kv > 0 ? a.N_kv : a.N;
  CUtensorMap mq, mk, mv;
  if (!make_map16(&mq, a.q, BH, a.N, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kTile) ||
      !make_map16(&mk, a.k_split, 2 * BH, N_kv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 64) ||
      !make_map16(&mv, a.v_f16, BH, N_kv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kTile))
    return -4;
  Params p;
  p.cos = a.cos;
  p.sin = a.sin;
  p.out = a.out;
  p.lse = a.lse;
  p.status = device_status_word();
  if (p.status == nullptr) return -4;
  p.BH = BH;
  p.N = a.N;
  p.N_kv = N_kv;
  p.n_kv = (N_kv + kTile - 1) / kTile;
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
    if (cudaFuncSetAttribute(attn_fwd_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, attn_fwd_split_kernel, mq, mk, mv, p) == cudaSuccess ? 0 : -4;
}

}  // namespace dit
