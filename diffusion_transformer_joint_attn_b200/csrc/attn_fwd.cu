// Joint text+image attention forward for sm_100a (BF16 in, BF16/fp32 out).
//
// One CTA owns two 128-row query tiles of one (b, h) and streams every
// 128-key tile of K and V past them (flash-style online softmax), so the
// logits never leave the SM.  Roles, by warp:
//
//   warp 0        TMA producer: Q tiles once, then K_j / V_j into 2-slot rings
//   warp 1        MMA issuer:   S_t = Q_t K_j^T (bf16 operands, smem x smem)
//                               O_t += P_t V_j (fp16 operands, P from TMEM)
//   warps 2-3,    operand prologue: rotary embedding of Q (once) and of every
//   12-15         K_j in shared memory (fp32 math, rounded to bf16), and the
//                 exact bf16 -> fp16 conversion of every V_j
//   warps 4-7     softmax of query tile 0 (one thread per query row)
//   warps 8-11    softmax of query tile 1
//
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1, each 128 lanes x 128
// fp32 columns; P_t (fp16) overwrites the first 64 columns of S_t.  While the
// softmax warps of one tile work, the tensor core runs the other tile's MMAs.
#include <cstdio>

#include "launch.h"
#include "ptx.cuh"
#include "rope_exact.cuh"

namespace dit {
namespace {

constexpr int kTile = 128;                  // query rows per tile = keys per tile
constexpr int kHeadDim = 128;
constexpr int kStages = 2;                  // K and V ring depth
constexpr int kTileBytes = kTile * kHeadDim * 2;   // 32 KB
constexpr int kBoxBytes = kTile * 64 * 2;          // 16 KB: 128 rows x 64 channels
constexpr int kThreads = 512;
constexpr int kProWarps = 6;
constexpr int kProThreads = kProWarps * 32;
constexpr int kChunks = kTileBytes / 16;           // 16-byte chunks per tile

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full;
  uint64_t q_ready;
  uint64_t k_full[kStages], k_ready[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_ready[kStages], v_empty[kStages];
  uint64_t s_full[2], p_ready[2], o_final[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  const float* cos;   // [N][64] or nullptr
  const float* sin;
  void* out;
  float* lse;
  int* status;
  int N;
  int n_qtiles;
  int n_kv;
  int pairs;          // query-tile pairs per (b, h)
  int out_f32;
  int rotate_k;       // rotate K tiles in the kernel (0: K arrives rotated or no rotary embedding)
  float scale_log2;   // log2(e) / sqrt(D)
};

// Byte offset, inside a tile, of 16-byte chunk `c` (0..2047) of the physical
// layout the 128-byte-swizzled TMA boxes produce, and the tile coordinates
// (row, first channel) whose 8 values it holds.
__device__ __forceinline__ void chunk_coords(int c, int& byte_off, int& row, int& col0) {
  const int box = c >> 10;          // channels 0-63 | 64-127
  row = (c >> 3) & 127;
  const int phys = c & 7;
  const int logical = phys ^ (row & 7);
  byte_off = box * kBoxBytes + row * 128 + phys * 16;
  col0 = box * 64 + logical * 8;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Rotate the pairs of one 128 x 128 bf16 tile in place, each result rounded
// exactly to bf16.  Row r is token n0+r; rows at or past N stay untouched.
__device__ __forceinline__ void rotate_tile(uint8_t* tile, int n0, const Params& p, int pt) {
  for (int c = pt; c < kChunks; c += kProThreads) {
    int off, row, col0;
    chunk_coords(c, off, row, col0);
    const int n = n0 + row;
    if (n >= p.N) continue;
    uint4 x = *reinterpret_cast<const uint4*>(tile + off);
    const int j0 = n * (kHeadDim / 2) + (col0 >> 1);
    const float4 cs = __ldg(reinterpret_cast<const float4*>(p.cos + j0));
    const float4 sn = __ldg(reinterpret_cast<const float4*>(p.sin + j0));
    x.x = rotate_pair_bf16(x.x, cs.x, sn.x);
    x.y = rotate_pair_bf16(x.y, cs.y, sn.y);
    x.z = rotate_pair_bf16(x.z, cs.z, sn.z);
    x.w = rotate_pair_bf16(x.w, cs.w, sn.w);
    *reinterpret_cast<uint4*>(tile + off) = x;
  }
}

// bf16 -> fp16 in place (exact for |x| in [2^-14, 65504]; below that the
// fp16 subnormal spacing 2^-24 bounds the error).
__device__ __forceinline__ void convert_tile_f16(uint8_t* tile, int pt) {
  for (int c = pt; c < kChunks; c += kProThreads) {
    uint4* ptr = reinterpret_cast<uint4*>(tile + c * 16);
    uint4 x = *ptr;
    x.x = pack_f16(bf16_lo(x.x), bf16_hi(x.x));
    x.y = pack_f16(bf16_lo(x.y), bf16_hi(x.y));
    x.z = pack_f16(bf16_lo(x.z), bf16_hi(x.z));
    x.w = pack_f16(bf16_lo(x.w), bf16_hi(x.w));
    *ptr = x;
  }
}

// TMA producer (warp 0).
__device__ __forceinline__ void producer_role(Smem& sm, const Params& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v, uint32_t tmem, int bh, int q0, int warp, int lane, const WaitCtx& wc) {
  if (lane == 0) {
    tma_prefetch_desc(tm_q);
    tma_prefetch_desc(tm_k);
    tma_prefetch_desc(tm_v);
    mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
    for (int t = 0; t < 2; ++t)
      for (int b = 0; b < 2; ++b) tma_load_3d(sm.q[t] + b * kBoxBytes, tm_q, &sm.q_full, b * 64, q0 + t * kTile, bh);
    int issued = 0;
    for (int j = 0; j < p.n_kv; ++j) {
      const int s = j % kStages;
      const uint32_t ph = (j / kStages) & 1;
      if (!mbar_wait(&sm.k_empty[s], ph ^ 1, wc)) break;
      mbar_arrive_expect_tx(&sm.k_full[s], kTileBytes);
      for (int b = 0; b < 2; ++b) tma_load_3d(sm.k[s] + b * kBoxBytes, tm_k, &sm.k_full[s], b * 64, j * kTile, bh);
      if (!mbar_wait(&sm.v_empty[s], ph ^ 1, wc)) {
        issued = 2 * j + 1;
        break;
      }
      mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
      for (int b = 0; b < 2; ++b) tma_load_3d(sm.v[s] + b * kBoxBytes, tm_v, &sm.v_full[s], b * 64, j * kTile, bh);
      issued = 2 * j + 2;
    }
    if (*wc.abort) {
      // let every copy already issued land before the CTA exits
      mbar_wait_drain(&sm.q_full, 0, wc);
      for (int i = (issued > 2 * kStages ? issued - 2 * kStages : 0); i < issued; ++i) {
        const int j = i / 2, s = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        mbar_wait_drain((i & 1) ? &sm.v_full[s] : &sm.k_full[s], ph, wc);
      }
    }
  }
}

// MMA issuer (warp 1).
__device__ __forceinline__ void mma_role(Smem& sm, const Params& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v, uint32_t tmem, int bh, int q0, int warp, int lane, const WaitCtx& wc) {
  if (lane == 0) {
    constexpr uint32_t idesc_qk = instr_desc(1, 1, 128, 128, 0, 0);   // bf16 x bf16, both K-major
    constexpr uint32_t idesc_pv = instr_desc(0, 0, 128, 128, 0, 1);   // f16 x f16, V MN-major
    const uint32_t q_addr[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
    bool ok = mbar_wait(&sm.q_ready, 0, wc);
    tc_fence_after();
    int j = 0;
    for (; ok && j <= p.n_kv; ++j) {
      const int s = j % kStages;
      const int sp = (j + kStages - 1) % kStages;
      for (int t = 0; t < 2 && ok; ++t) {
        const uint32_t tS = tmem + t * 128;
        const uint32_t tO = tmem + 256 + t * 128;
        if (j > 0) {
          // O_t += P_t V_{j-1}
          if (!(ok = mbar_wait(&sm.p_ready[t], (j - 1) & 1, wc))) break;
          if (t == 0 && !(ok = mbar_wait(&sm.v_ready[sp], ((j - 1) / kStages) & 1, wc))) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sm.v[sp]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 2048, kBoxBytes, 1024);
            mma_ts(tO, tS + kk * 8, bdesc, idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
          }
          if (j == p.n_kv) tc_commit(&sm.o_final[t]);
        }
        if (j < p.n_kv) {
          // S_t = Q_t K_j^T
          if (t == 0) {
            if (!(ok = mbar_wait(&sm.k_ready[s], (j / kStages) & 1, wc))) break;
            tc_fence_after();
          }
          const uint32_t k_addr = smem_u32(sm.k[s]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
            const uint64_t adesc = smem_desc_sw128(q_addr[t] + off, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(k_addr + off, 16, 1024);
            mma_ss(tS, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(&sm.s_full[t]);
        }
      }
      if (!ok) break;
      if (j < p.n_kv) tc_commit(&sm.k_empty[s]);
      if (j > 0) tc_commit(&sm.v_empty[sp]);
    }
    // every MMA issued above has completed once this arrives
    tc_commit(&sm.mma_drain);
    mbar_wait_drain(&sm.mma_drain, 0, wc);
  }
}

// Online softmax and epilogue of one query tile (warps 4-11).
__device__ __forceinline__ void softmax_role(Smem& sm, const Params& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v, uint32_t tmem, int bh, int q0, int warp, int lane, const WaitCtx& wc) {
  const int t = (warp - 4) >> 2;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + t * 128;
  const uint32_t tO = tmem + lane_base + 256 + t * 128;
  const float c = p.scale_log2;
  const float rescale_gap = 8.0f / c;     // lazy rescale once the max grew by 2^8
  const int last_valid = p.N - (p.n_kv - 1) * kTile;
  float m_used = 0.f, l = 0.f;
  bool ok = true;
  for (int j = 0; j < p.n_kv; ++j) {
    if (!(ok = warp_wait(&sm.s_full[t], j & 1, wc))) break;
    tc_fence_after();
    uint32_t s[128];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, s + q * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld_wait(s + q * 32);
    float* f = reinterpret_cast<float*>(s);
    if (j == p.n_kv - 1 && last_valid < kTile) {
#pragma unroll
      for (int i = 0; i < 128; ++i)
        if (i >= last_valid) f[i] = -INFINITY;
    }
    float mx = f[0];
#pragma unroll
    for (int i = 1; i < 128; ++i) mx = fmaxf(mx, f[i]);
    // Lazy rescale: keep the stale maximum unless it grew by more than 2^8
    // (P then stays <= 256); the decision is warp-uniform because the O
    // rescale uses warp-collective TMEM loads/stores.
    float alpha = 1.0f;
    bool rescale = false;
    if (j == 0) {
      m_used = mx;
    } else if (__any_sync(0xffffffffu, mx > m_used + rescale_gap)) {
      const float m_new = fmaxf(m_used, mx);
      alpha = ex2_approx((m_used - m_new) * c);
      m_used = m_new;
      l *= alpha;
      rescale = true;
    }
    const float neg = -m_used * c;
    float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = ex2_approx(fmaf(f[64 * h + 2 * i], c, neg));
        const float p1 = ex2_approx(fmaf(f[64 * h + 2 * i + 1], c, neg));
        pk[i] = pack_f16(p0, p1);
        // l sums the fp16-rounded P the MMA multiplies V with, so a row
        // dominated by one key returns that key's V row exactly
        if (i & 1)
          sum1 = add_f16x2_to_f32(sum1, pk[i]);
        else
          sum0 = add_f16x2_to_f32(sum0, pk[i]);
      }
      tmem_st32(tS + 32 * h, pk);
    }
    l += sum0 + sum1;
    if (rescale) {
      // O_t holds P V up to tile j-1 (that MMA completed before S_t of
      // tile j was committed) and no MMA writes it until p_ready.
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + q * 32, o);
        tmem_ld_wait(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        tmem_st32(tO + q * 32, o);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.p_ready[t]);
  }
  // epilogue: O / l and the log-sum-exp
  if (ok && warp_wait(&sm.o_final[t], 0, wc)) {
    tc_fence_after();
    const int n = q0 + t * kTile + row;
    const bool valid = n < p.N;
    const float inv_l = 1.0f / l;
    const size_t row_off = (static_cast<size_t>(bh) * p.N + n) * kHeadDim;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t o[32];
      tmem_ld32(tO + q * 32, o);
      tmem_ld_wait(o);
      if (valid) {
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row_off + q * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                 __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row_off + q * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float* v8 = reinterpret_cast<const float*>(o + 8 * i);
            dst[i] = make_uint4(pack_bf16(v8[0] * inv_l, v8[1] * inv_l), pack_bf16(v8[2] * inv_l, v8[3] * inv_l),
                                pack_bf16(v8[4] * inv_l, v8[5] * inv_l), pack_bf16(v8[6] * inv_l, v8[7] * inv_l));
          }
        }
      }
    }
    if (valid && p.lse != nullptr) {
      p.lse[static_cast<size_t>(bh) * p.N + n] = (m_used * c + lg2_approx(l)) * 0.69314718055994530942f;
    }
  }
}

// Operand prologue: rotary embedding of Q / K, fp16 conversion of V (warps 2-3, 12-15).
__device__ __forceinline__ void prologue_role(Smem& sm, const Params& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v, uint32_t tmem, int bh, int q0, int warp, int lane, const WaitCtx& wc) {
  const int pt = (warp < 4 ? (warp - 2) * 32 : 64 + (warp - 12) * 32) + lane;
  const bool rope = p.cos != nullptr;
  if (warp_wait(&sm.q_full, 0, wc)) {
    if (rope) {
      rotate_tile(sm.q[0], q0, p, pt);
      rotate_tile(sm.q[1], q0 + kTile, p, pt);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.q_ready);
    for (int j = 0; j < p.n_kv; ++j) {
      const int s = j % kStages;
      const uint32_t ph = (j / kStages) & 1;
      if (!warp_wait(&sm.k_full[s], ph, wc)) break;
      if (rope && p.rotate_k) rotate_tile(sm.k[s], j * kTile, p, pt);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.k_ready[s]);
      if (!warp_wait(&sm.v_full[s], ph, wc)) break;
      convert_tile_f16(sm.v[s], pt);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.v_ready[s]);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.pairs;
  const int q0 = (blockIdx.x % p.pairs) * 2 * kTile;
  const WaitCtx wc{&sm.abort, p.status};

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_ready, kProWarps);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_ready[s], kProWarps);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_ready[s], kProWarps);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_ready[t], 4);
      mbar_init(&sm.o_final[t], 1);
    }
    mbar_init(&sm.mma_drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // 4 warpgroups share 4 x 128 x 128 registers: the two softmax warpgroups
  // take 192 per thread, the producer / MMA / prologue warpgroups keep 64.
  const int wg = warp >> 2;
  if (wg == 1 || wg == 2) {
    regs_increase<192>();
    softmax_role(sm, p, &tm_q, &tm_k, &tm_v, tmem, bh, q0, warp, lane, wc);
  } else {
    regs_decrease<64>();
    if (warp == 0)
      producer_role(sm, p, &tm_q, &tm_k, &tm_v, tmem, bh, q0, warp, lane, wc);
    else if (warp == 1)
      mma_role(sm, p, &tm_q, &tm_k, &tm_v, tmem, bh, q0, warp, lane, wc);
    else
      prologue_role(sm, p, &tm_q, &tm_k, &tm_v, tmem, bh, q0, warp, lane, wc);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

bool make_map(CUtensorMap* map, const void* base, int BH, int N) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                 static_cast<cuuint64_t>(N) * kHeadDim * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTile), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int launch_attn_fwd_bf16(const AttnFwdArgs& a, cudaStream_t s) {
  const int BH = a.B * a.H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, BH, a.N) || !make_map(&mk, a.k, BH, a.N) || !make_map(&mv, a.v, BH, a.N)) return -4;
  Params p;
  p.cos = a.cos;
  p.sin = a.sin;
  p.out = a.out;
  p.lse = a.lse;
  p.status = device_status_word();
  if (p.status == nullptr) return -4;
  p.N = a.N;
  p.n_qtiles = (a.N + kTile - 1) / kTile;
  p.n_kv = p.n_qtiles;
  p.pairs = (p.n_qtiles + 1) / 2;
  p.out_f32 = a.out_f32 ? 1 : 0;
  p.rotate_k = (a.cos != nullptr && !a.k_rotated) ? 1 : 0;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kHeadDim));
  const size_t smem = sizeof(Smem) + 1024;
  static thread_local int configured_device = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -4;
  if (configured_device != dev) {
    if (cudaFuncSetAttribute(attn_fwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -4;
    configured_device = dev;
  }
  const long long grid = static_cast<long long>(BH) * p.pairs;
  if (grid > 0x7FFFFFFFLL) return -1;
  attn_fwd_bf16_kernel<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace dit
