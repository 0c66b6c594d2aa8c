// Joint text+image attention forward for sm_100a (BF16 in, BF16/fp32 out).
//
// A cluster of two CTAs (a CTA pair on the two SMs of a TPC) owns four
// 128-row query tiles of one (b, h): two per CTA, processed as two 256-row
// "slots" (rows 0-127 of a slot in the even CTA, 128-255 in the odd one).
// Every 128-key tile of K and V streams past them (flash-style online
// softmax), so the logits never leave the SMs.  The even CTA issues pair MMAs
// (tcgen05 cta_group::2, M = 256) that read each CTA's own Q rows and P rows
// and half of the B operand from each CTA: keys 0-63 / 64-127 of a K tile,
// channels 0-63 / 64-127 of a V tile.  Each SM therefore loads and reads
// only half of every K and V tile, which keeps the shared-memory port below
// the rate the two products need.
//
// Roles, by warp (in both CTAs unless stated):
//   warp 0        TMA producer: own Q tiles once, own K_j / V_j halves into
//                 4-slot rings
//   warp 1        MMA issuer (even CTA only): S_t = Q_t K_j^T (bf16),
//                 O_t += P_t V_j (fp16, P from tensor memory)
//   warps 2-11    rotary embedding of the CTA's two Q tiles, once (and
//   (2-15)        warps 12-15 where they exist)
//   warps 2-3,    in-loop operand work when K / V were not prepared by
//   12-15         dit_attn_prepare_kv: rotation of the K_j half and the exact
//                 bf16 -> fp16 conversion of the V_j half, in shared memory
//   warps 4-7     softmax of slot 0 (one thread per query row)
//   warps 8-11    softmax of slot 1
//
// On prepared operands the CTA has 12 warps: 65536 / 384 threads leaves 168
// registers per thread, enough for a softmax thread's 128 logits, so no
// register reallocation is needed.  With in-loop operand work it has 16
// warps, and setmaxnreg moves registers from warpgroups 0 and 3 to the
// softmax warpgroups.  Only that instance contains setmaxnreg: measured on
// the B200, a kernel that contains it (even unexecuted) issues the pair MMAs
// of this loop at 74-86 % of the rate of the same kernel without it.
//
// Tensor memory per CTA (512 columns): S_0 | S_1 | O_0 | O_1, 128 lanes x 128
// fp32 columns each; P_t (fp16) overwrites the first 64 columns of S_t.
// While the softmax warps of one slot work, the tensor cores run the other
// slot's MMAs.
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

constexpr int kStages = 4;                         // K and V ring depth
constexpr int kQTileBytes = kTile * kHeadDim * 2;  // 32 KB: 128 rows x 128 channels
constexpr int kQBoxBytes = kTile * 64 * 2;         // 16 KB: 128 rows x 64 channels
constexpr int kKHalfBytes = 64 * kHeadDim * 2;     // 16 KB: 64 keys x 128 channels
constexpr int kKBoxBytes = 64 * 64 * 2;            // 8 KB: 64 keys x 64 channels
constexpr int kVHalfBytes = kTile * 64 * 2;        // 16 KB: 128 keys x 64 channels
// Threads per CTA: 12 warps on prepared operands, 16 with in-loop operand work.
template <bool kPrepared>
constexpr int kThreadsOf = kPrepared ? 384 : 512;
constexpr int kProWarps = 6;                       // in-loop operand warps per CTA
constexpr int kProThreads = kProWarps * 32;
constexpr int kBarQRot = 1;                        // named barrier of the Q rotation
constexpr int kMaxKvTiles = 4096;                  // block-sparse launches: N <= 4096 x 128 keys
// Register split of the 4 x 128 x 128 launch registers of the 16-warp CTA
// between warpgroups: producer / MMA warpgroup, the two softmax warpgroups,
// the operand warpgroup.
constexpr uint32_t kIssueRegs = 80;
constexpr uint32_t kSoftmaxRegs = 184;
constexpr uint32_t kOperandRegs = 64;
static_assert(kIssueRegs + 2 * kSoftmaxRegs + kOperandRegs == 4 * 128, "register split must use the launch budget");

struct __align__(1024) Smem {
  uint8_t q[2][kQTileBytes];
  uint8_t k[kStages][kKHalfBytes];
  uint8_t v[kStages][kVHalfBytes];
  uint64_t q_full;
  uint64_t q_ready;                                   // even CTA: one arrive per CTA
  uint64_t k_full[kStages], k_ready[kStages];
  uint64_t v_full[kStages], v_ready[kStages];
  uint64_t kv_empty[kStages];                          // stage s free again: P V of its tile has completed
  uint64_t s_full[2], p_ready[2], o_final[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
  int n_act;                                           // key tiles this pair attends to
  // block-sparse launches: the tiles' indices (uint16_t[kMaxKvTiles]) follow the struct
};

struct Params {
  const float* cos;   // [N][64] or nullptr
  const float* sin;
  void* out;
  float* lse;
  int* status;
  const uint8_t* kv_mask;   // [B*H][clusters][n_kv] block mask, or nullptr (all key tiles)
  int N;              // query rows per (b, h)
  int N_kv;           // keys per (b, h)
  int n_kv;
  int clusters;       // CTA pairs per (b, h): 512 query rows each
  int out_f32;
  int rotate_k;       // rotate K halves in the loop
  int convert_v;      // convert V halves bf16 -> fp16 in the loop
  float scale_log2;   // log2(e) / sqrt(D)
};

// Block-sparse launches keep the pair's list of key tiles right after Smem.
__device__ __forceinline__ uint16_t* kv_list(Smem& sm) { return reinterpret_cast<uint16_t*>(&sm + 1); }
__device__ __forceinline__ const uint16_t* kv_list(const Smem& sm) {
  return reinterpret_cast<const uint16_t*>(&sm + 1);
}

// Key tile visited at step i: the i-th tile of the pair's list (kSparse),
// else tile i.  Number of steps: the list's length, else all n_kv tiles.
template <bool kSparse>
__device__ __forceinline__ int kv_tile(const Smem& sm, int i) {
  return kSparse ? static_cast<int>(kv_list(sm)[i]) : i;
}
template <bool kSparse>
__device__ __forceinline__ int kv_steps(const Smem& sm, const Params& p) {
  return kSparse ? sm.n_act : p.n_kv;
}

// Compact the pair's row of the block mask into the tile list and n_act (one
// warp; both CTAs of the pair read the same row).
__device__ __forceinline__ void build_kv_list(Smem& sm, const Params& p, const Pair& pr, int qblock, int lane) {
  const uint8_t* row = p.kv_mask + (static_cast<size_t>(pr.bh) * p.clusters + qblock) * p.n_kv;
  uint16_t* list = kv_list(sm);
  int count = 0;
  for (int base = 0; base < p.n_kv; base += 32) {
    const int tile = base + lane;
    const bool on = tile < p.n_kv && row[tile] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (on) list[count + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(tile);
    count += __popc(bal);
  }
  if (lane == 0) sm.n_act = count;
}

// Q tile chunk c (0..2047): byte offset in the 128B-swizzled layout of two
// 128-row x 64-channel boxes, its row and first channel.
__device__ __forceinline__ void q_chunk(int c, int& byte_off, int& row, int& col0) {
  const int box = c >> 10;
  row = (c >> 3) & 127;
  const int phys = c & 7;
  byte_off = box * kQBoxBytes + row * 128 + phys * 16;
  col0 = box * 64 + ((phys ^ (row & 7)) << 3);
}
// K half-tile chunk c (0..1023): two 64-row x 64-channel boxes.
__device__ __forceinline__ void k_chunk(int c, int& byte_off, int& row, int& col0) {
  const int box = c >> 9;
  row = (c >> 3) & 63;
  const int phys = c & 7;
  byte_off = box * kKBoxBytes + row * 128 + phys * 16;
  col0 = box * 64 + ((phys ^ (row & 7)) << 3);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Rotate chunks first, first+kStep, ... (< kChunks) of a tile whose row r is
// token n0 + r, in place, each component rounded exactly to bf16.  The loads
// of kBatch chunks are issued before any of them is used.
template <int kChunks, int kStep, int kBatch, bool kHalfK>
__device__ __forceinline__ void rotate_chunks(uint8_t* tile, int n0, const Params& p, int first) {
  for (int c0 = first; c0 < kChunks; c0 += kBatch * kStep) {
    uint4 x[kBatch];
    float4 cs[kBatch], sn[kBatch];
    int off[kBatch];
    bool live[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int c = c0 + u * kStep;
      int row, col0;
      if (kHalfK)
        k_chunk(c < kChunks ? c : 0, off[u], row, col0);
      else
        q_chunk(c < kChunks ? c : 0, off[u], row, col0);
      const int n = n0 + row;
      live[u] = c < kChunks && n < (kHalfK ? p.N_kv : p.N);
      if (live[u]) {
        const int j0 = n * (kHeadDim / 2) + (col0 >> 1);
        x[u] = *reinterpret_cast<const uint4*>(tile + off[u]);
        cs[u] = __ldg(reinterpret_cast<const float4*>(p.cos + j0));
        sn[u] = __ldg(reinterpret_cast<const float4*>(p.sin + j0));
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (!live[u]) continue;
      uint4 y;
      y.x = rotate_pair_bf16(x[u].x, cs[u].x, sn[u].x);
      y.y = rotate_pair_bf16(x[u].y, cs[u].y, sn[u].y);
      y.z = rotate_pair_bf16(x[u].z, cs[u].z, sn[u].z);
      y.w = rotate_pair_bf16(x[u].w, cs[u].w, sn[u].w);
      *reinterpret_cast<uint4*>(tile + off[u]) = y;
    }
  }
}

// bf16 -> fp16 in place for a V half tile (exact for |x| in [2^-14, 65504];
// below that the fp16 subnormal spacing 2^-24 bounds the error).
__device__ __forceinline__ void convert_half_f16(uint8_t* tile, int pt) {
  for (int c = pt; c < kVHalfBytes / 16; c += kProThreads) {
    uint4* ptr = reinterpret_cast<uint4*>(tile + c * 16);
    uint4 x = *ptr;
    x.x = pack_f16(bf16_lo(x.x), bf16_hi(x.x));
    x.y = pack_f16(bf16_lo(x.y), bf16_hi(x.y));
    x.z = pack_f16(bf16_lo(x.z), bf16_hi(x.z));
    x.w = pack_f16(bf16_lo(x.w), bf16_hi(x.w));
    *ptr = x;
  }
}

// ---------------------------------------------------------------- producer
// kPrepared: K / V halves land MMA-ready; their bytes are counted on the even
// CTA's barriers (one expect_tx there covers both halves).  Otherwise each
// CTA counts its own halves locally for its operand warps.
template <bool kPrepared, bool kSparse>
__device__ __forceinline__ void producer_role(Smem& sm, const Params& p, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k, const CUtensorMap* tm_v, const Pair& pr,
                                              const WaitCtx& wc) {
  tma_prefetch_desc(tm_q);
  tma_prefetch_desc(tm_k);
  tma_prefetch_desc(tm_v);
  mbar_arrive_expect_tx(&sm.q_full, 2 * kQTileBytes);
  for (int t = 0; t < 2; ++t)
    for (int b = 0; b < 2; ++b)
      tma_load_3d(sm.q[t] + b * kQBoxBytes, tm_q, &sm.q_full, b * 64, pr.row0[t], pr.bh);
  const bool leader = pr.rank == 0;
  int issued = 0;
  const int steps = kv_steps<kSparse>(sm, p);
  for (int j = 0; j < steps; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (j / kStages) & 1;
    const int key0 = kv_tile<kSparse>(sm, j) * kTile;
    if (!mbar_wait(&sm.kv_empty[s], ph ^ 1, wc)) break;
    if (kPrepared) {
      if (leader) mbar_arrive_expect_tx(&sm.k_full[s], 2 * kKHalfBytes);
      const uint32_t bar = cl(&sm.k_full[s], 0);
      for (int b = 0; b < 2; ++b)
        tma_load_3d_pair(sm.k[s] + b * kKBoxBytes, tm_k, bar, b * 64, key0 + 64 * static_cast<int>(pr.rank), pr.bh);
    } else {
      mbar_arrive_expect_tx(&sm.k_full[s], kKHalfBytes);
      for (int b = 0; b < 2; ++b)
        tma_load_3d(sm.k[s] + b * kKBoxBytes, tm_k, &sm.k_full[s], b * 64, key0 + 64 * static_cast<int>(pr.rank),
                    pr.bh);
    }
    if (kPrepared) {
      if (leader) mbar_arrive_expect_tx(&sm.v_full[s], 2 * kVHalfBytes);
      tma_load_3d_pair(sm.v[s], tm_v, cl(&sm.v_full[s], 0), 64 * static_cast<int>(pr.rank), key0, pr.bh);
    } else {
      mbar_arrive_expect_tx(&sm.v_full[s], kVHalfBytes);
      tma_load_3d(sm.v[s], tm_v, &sm.v_full[s], 64 * static_cast<int>(pr.rank), key0, pr.bh);
    }
    issued = 2 * j + 2;
  }
  if (*wc.abort) {
    // Let the copies already issued land before the pair exits.  Copies whose
    // bytes the even CTA counts are drained there; the odd CTA waits out a
    // few microseconds instead.
    mbar_wait_drain(&sm.q_full, 0, wc);
    if (!kPrepared || leader) {
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

// ---------------------------------------------------------------- MMA issuer
// Even CTA only.  Completion of pair MMAs is signalled to the barrier of the
// same name in both CTAs.
template <bool kPrepared, bool kSparse>
__device__ __forceinline__ void mma_role(Smem& sm, const Params& p, uint32_t tmem, const WaitCtx& wc) {
  constexpr uint32_t idesc_qk = instr_desc(1, 1, 256, 128, 0, 0);   // bf16 x bf16, both K-major
  constexpr uint32_t idesc_pv = instr_desc(0, 0, 256, 128, 0, 1);   // f16 x f16, V MN-major
  // Descriptors, built once: ring slots are contiguous, so slot s and the k-th
  // 16-wide slice of a tile only move the start address (field in 16-byte
  // units) by constants; no runtime-indexed arrays (they would live in local
  // memory and stall the issuing thread).
  const uint64_t q_desc0 = smem_desc_sw128(smem_u32(sm.q[0]), 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(smem_u32(sm.k[0]), 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(smem_u32(sm.v[0]), kVHalfBytes, 1024);
  uint64_t* k_bar = kPrepared ? sm.k_full : sm.k_ready;
  uint64_t* v_bar = kPrepared ? sm.v_full : sm.v_ready;
  bool ok = mbar_wait(&sm.q_ready, 0, wc);
  tc_fence_after();
  const int n_act = kv_steps<kSparse>(sm, p);
  for (int j = 0; ok && j <= n_act; ++j) {
    const int s = j % kStages;
    const int sp = (j + kStages - 1) % kStages;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t tS = tmem + t * 128;
      const uint32_t tO = tmem + 256 + t * 128;
      if (j > 0) {
        // O_t += P_t V_{j-1}
        if (!(ok = mbar_wait(&sm.p_ready[t], (j - 1) & 1, wc))) break;
        if (t == 0 && !(ok = mbar_wait(&v_bar[sp], ((j - 1) / kStages) & 1, wc))) break;
        tc_fence_after();
        const uint64_t vd = v_desc0 + static_cast<uint32_t>(sp) * (kVHalfBytes >> 4);
        mma_ts_pair(tO, tS, vd, idesc_pv, j > 1 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) mma_ts_pair(tO, tS + kk * 8, vd + kk * (2048 >> 4), idesc_pv, 1u);
        if (j == n_act) commit_both(&sm.o_final[t]);
      }
      if (j < n_act) {
        // S_t = Q_t K_j^T
        if (t == 0) {
          if (!(ok = mbar_wait(&k_bar[s], (j / kStages) & 1, wc))) break;
          tc_fence_after();
        }
        const uint64_t qd = q_desc0 + t * (kQTileBytes >> 4);
        const uint64_t kd = k_desc0 + static_cast<uint32_t>(s) * (kKHalfBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = ((kk >> 2) * kQBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t boff = ((kk >> 2) * kKBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss_pair(tS, qd + aoff, kd + boff, idesc_qk, kk > 0 ? 1u : 0u);
        }
        commit_both(&sm.s_full[t]);
      }
    }
    if (!ok) break;
    // one release per stage: the commit tracks Q K_{j-1}^T and P V_{j-1}
    if (j > 0) commit_both(&sm.kv_empty[sp]);
  }
  if (kSparse && ok && n_act == 0) {   // no key tile: nothing to wait for
    commit_both(&sm.o_final[0]);
    commit_both(&sm.o_final[1]);
  }
  // every MMA issued above has completed once this arrives
  tc_commit_pair(cl(&sm.mma_drain, 0));
  mbar_wait_drain(&sm.mma_drain, 0, wc);
}

// ---------------------------------------------------------------- operand work
// Rotary embedding of the CTA's two Q tiles by warps 2 .. (kRotThreads / 32
// + 1), then one arrive on the even CTA's q_ready.  kBatch: loads in flight
// per thread.
template <int kBatch, int kRotThreads>
__device__ __forceinline__ void rotate_q(Smem& sm, const Params& p, const Pair& pr, int warp, int lane,
                                         const WaitCtx& wc) {
  const int qt = (warp - 2) * 32 + lane;      // 0 .. kRotThreads - 1
  const bool ok = warp_wait(&sm.q_full, 0, wc);
  if (ok && p.cos != nullptr) {
    rotate_chunks<kQTileBytes / 16, kRotThreads, kBatch, false>(sm.q[0], pr.row0[0], p, qt);
    rotate_chunks<kQTileBytes / 16, kRotThreads, kBatch, false>(sm.q[1], pr.row0[1], p, qt);
  }
  fence_proxy_async_smem();
  named_bar_sync(kBarQRot, kRotThreads);
  if (ok && qt == 0) mbar_arrive_cluster(cl(&sm.q_ready, 0));
}

// In-loop operand work (warps 2-3, 12-15) on this CTA's K_j and V_j halves.
template <bool kSparse>
__device__ __forceinline__ void kv_prologue_role(Smem& sm, const Params& p, const Pair& pr, int warp, int lane,
                                                 const WaitCtx& wc) {
  const int pt = (warp < 4 ? (warp - 2) * 32 : 64 + (warp - 12) * 32) + lane;
  const int steps = kv_steps<kSparse>(sm, p);
  for (int j = 0; j < steps; ++j) {
    const int s = j % kStages;
    const uint32_t ph = (j / kStages) & 1;
    if (!warp_wait(&sm.k_full[s], ph, wc)) break;
    if (p.rotate_k)
      rotate_chunks<kKHalfBytes / 16, kProThreads, 2, true>(sm.k[s],
                                                            kv_tile<kSparse>(sm, j) * kTile + 64 * static_cast<int>(pr.rank),
                                                            p, pt);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(cl(&sm.k_ready[s], 0));
    if (!warp_wait(&sm.v_full[s], ph, wc)) break;
    if (p.convert_v) convert_half_f16(sm.v[s], pt);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(cl(&sm.v_ready[s], 0));
  }
}

template <bool kPrepared, bool kSparse>
__global__ void __launch_bounds__(kThreadsOf<kPrepared>, 1)
    attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
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
      mbar_init(&sm.k_ready[s], 2 * kProWarps);
      mbar_init(&sm.kv_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_ready[s], 2 * kProWarps);
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
  if (kSparse && warp == 2) build_kv_list(sm, p, pr, cluster % p.clusters, lane);
  tc_fence_before();
  cluster_sync();          // both CTAs' barriers initialised, tensor memory allocated, key list built
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort, p.status, cl(&sm.abort, pr.peer)};

  constexpr int kRotThreads = kThreadsOf<kPrepared> - 64;   // warps 2 and up
  const int wg = warp >> 2;
  if (wg == 1 || wg == 2) {
    if constexpr (!kPrepared) regs_increase<kSoftmaxRegs>();
    rotate_q<4, kRotThreads>(sm, p, pr, warp, lane, wc);
    attn::SoftmaxIo io{sm.s_full, sm.p_ready, sm.o_final, p.out, p.lse, p.N, p.N_kv, p.n_kv, p.out_f32,
                       p.scale_log2, nullptr, nullptr, 0, kv_list(sm), kv_steps<kSparse>(sm, p)};
    attn::softmax_slot<false, kSparse>(io, tmem, pr, warp, lane, wc);
  } else {
    if constexpr (!kPrepared) {
      if (wg == 0)
        regs_decrease<kIssueRegs>();
      else
        regs_decrease<kOperandRegs>();
    }
    if (warp == 0) {
      if (lane == 0) producer_role<kPrepared, kSparse>(sm, p, &tm_q, &tm_k, &tm_v, pr, wc);
    } else if (warp == 1) {
      if (lane == 0 && pr.rank == 0) mma_role<kPrepared, kSparse>(sm, p, tmem, wc);
    } else {
      rotate_q<2, kRotThreads>(sm, p, pr, warp, lane, wc);
      if constexpr (!kPrepared) kv_prologue_role<kSparse>(sm, p, pr, warp, lane, wc);
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();          // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

bool make_map(CUtensorMap* map, const void* base, int BH, int N, bool f16, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                 static_cast<cuuint64_t>(N) * kHeadDim * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kPrepared, bool kSparse>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p, long long grid,
           cudaStream_t s) {
  const size_t smem = sizeof(Smem) + (kSparse ? kMaxKvTiles * sizeof(uint16_t) : 0) + 1024;
  static thread_local int configured_device = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -4;
  if (configured_device != dev) {
    if (cudaFuncSetAttribute(attn_fwd_bf16_kernel<kPrepared, kSparse>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -4;
    configured_device = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreadsOf<kPrepared>, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_fwd_bf16_kernel<kPrepared, kSparse>, mq, mk, mv, p) == cudaSuccess ? 0 : -4;
}

}  // namespace

int launch_attn_fwd_bf16(const AttnFwdArgs& a, cudaStream_t s) {
  const int BH = a.B * a.H;
  const int N_kv = a.N_kv > 0 ? a.N_kv : a.N;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, BH, a.N, false, kTile) || !make_map(&mk, a.k, BH, N_kv, false, 64) ||
      !make_map(&mv, a.v, BH, N_kv, a.v_f16, kTile))
    return -4;
  Params p;
  p.cos = a.cos;
  p.sin = a.sin;
  p.out = a.out;
  p.lse = a.lse;
  p.status = device_status_word();
  if (p.status == nullptr) return -4;
  p.kv_mask = a.kv_mask;
  p.N = a.N;
  p.N_kv = N_kv;
  p.n_kv = (N_kv + kTile - 1) / kTile;
  if (a.kv_mask != nullptr && p.n_kv > kMaxKvTiles) return -2;
  p.clusters = (a.N + 4 * kTile - 1) / (4 * kTile);
  p.out_f32 = a.out_f32 ? 1 : 0;
  p.rotate_k = (a.cos != nullptr && !a.k_rotated) ? 1 : 0;
  p.convert_v = a.v_f16 ? 0 : 1;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kHeadDim));
  const long long grid = 2LL * BH * p.clusters;
  if (grid > 0x7FFFFFFFLL) return -1;
  const bool prepared = !p.rotate_k && !p.convert_v;
  if (a.kv_mask != nullptr)
    return prepared ? launch<true, true>(mq, mk, mv, p, grid, s) : launch<false, true>(mq, mk, mv, p, grid, s);
  return prepared ? launch<true, false>(mq, mk, mv, p, grid, s) : launch<false, false>(mq, mk, mv, p, grid, s);
}

}  // namespace dit
