// Device pieces shared by the BF16 and FP8 joint-attention kernels: CTA-pair
// addressing, the per-slot online softmax and the epilogue.
#pragma once

#include "ptx.cuh"
#include "rope_exact.cuh"
#include "softmax_exp2.cuh"

namespace dit {
namespace attn {

constexpr int kTile = 128;                         // query rows per tile = keys per K/V tile
constexpr int kHeadDim = 128;
// Every kPolyEvery-th exponent pair runs on the FMA pipe (0: none), per
// kernel: measured best at one pair in four for the BF16 kernel and one in
// three for the FP8 kernel (whose shorter Q K^T leaves the softmax less time).
template <bool kScaled>
constexpr int kPolyEvery = kScaled ? 3 : 4;

struct Pair {
  uint32_t rank;      // 0: even (MMA-issuing) CTA, 1: odd CTA
  uint32_t peer;
  int bh;
  int row0[2];        // first query row of this CTA's tile in slot 0 / 1
};

// shared::cluster address of `p` in CTA `rank` of the pair.
__device__ __forceinline__ uint32_t cl(const void* p, uint32_t rank) { return mapa_shared(smem_u32(p), rank); }

// Signal a pair-MMA completion to the barrier of the same name in both CTAs.
__device__ __forceinline__ void commit_both(uint64_t* bar) {
  tc_commit_pair(cl(bar, 0));
  tc_commit_pair(cl(bar, 1));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max of exactly the 64 values f[0..63] (4 independent chains of 3-input max;
// chain u takes elements 8i + 2u and 8i + 2u + 1).
__device__ __forceinline__ float max64(const float* f) {
  float m[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) m[u] = fmaxf(f[2 * u], f[2 * u + 1]);
#pragma unroll
  for (int i = 8; i < 64; i += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u) m[u] = fmax3(m[u], f[i + 2 * u], f[i + 2 * u + 1]);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Max of exactly the 128 values f[0..127] (4 chains of 3-input max).
__device__ __forceinline__ float max128(const float* f) {
  float m[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) m[u] = fmaxf(f[2 * u], f[2 * u + 1]);
#pragma unroll
  for (int i = 8; i < 128; i += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u) m[u] = fmax3(m[u], f[i + 2 * u], f[i + 2 * u + 1]);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// P for 2 kPairs consecutive logits of the row: 2^(s c - m c) rounded to
// fp16, packed in pairs into pk[kPairs]; adds the rounded values to sum[4].
template <int kPairs, int kPoly>
__device__ __forceinline__ void exp_pairs(const float* f, float c, float neg, uint32_t* pk, float* sum) {
  const float2 c2 = make_float2(c, c), n2 = make_float2(neg, neg);
#pragma unroll
  for (int i = 0; i < kPairs; ++i) {
    const float2 x = __ffma2_rn(make_float2(f[2 * i], f[2 * i + 1]), c2, n2);
    float e0, e1;
    if (kPoly > 0 && i % kPoly == kPoly - 1) {
      exp2_pair_poly(x.x, x.y, e0, e1);
    } else {
      e0 = ex2_approx(x.x);
      e1 = ex2_approx(x.y);
    }
    pk[i] = pack_f16(e0, e1);
    // l sums the fp16-rounded P the MMA multiplies V with, so a row
    // dominated by one key returns that key's V row exactly
    sum[i & 3] = add_f16x2_to_f32(sum[i & 3], pk[i]);
  }
}
template <int kPoly>
__device__ __forceinline__ void exp_half(const float* f, float c, float neg, uint32_t* pk, float* sum) {
  exp_pairs<32, kPoly>(f, c, neg, pk, sum);
}

// Barriers, outputs and (FP8 only) block scales of one CTA's softmax warps.
struct SoftmaxIo {
  uint64_t* s_full;        // [2] local: S_t of the current key tile is in tensor memory
  uint64_t* p_ready;       // [2] the even CTA's barriers count one arrive per softmax warp of the pair
  uint64_t* o_final;       // [2] local: the last P V product of slot t has completed
  void* out;
  float* lse;
  int N;                   // query rows per (b, h)
  int N_kv;                // keys per (b, h)
  int n_kv;                // key tiles: ceil(N_kv / 128)
  int out_f32;
  float scale_log2;        // log2(e) / sqrt(D)
  const float* q_scale;    // this (b, h)'s per-64-token scales, or nullptr (unscaled logits)
  const float* k_scale;
  int n_blocks;            // ceil(N / 64)
  const uint16_t* kv_list; // key tiles visited, in order (block-sparse instances only)
  int n_act;               // number of key tiles visited
};

// Online softmax of this CTA's tile of slot t, then the epilogue (warps 4-11).
//
// Logits are q~.k~ times an optional per-(query block, key block) factor
// (the FP8 operands' scales): within a 128-key tile the first and second 64
// keys have their own factor, folded into the exponent's fused multiply-add.
// The running maximum is kept lazily: P = 2^((s - m_used) c) with m_used
// raised only when a tile's maximum exceeds it by more than 15 (log2 units),
// so P stays in [0, 2^15], below the fp16 maximum (fp16 rounding is relative,
// so the size of P costs no precision, and a higher threshold means fewer
// rescales of O on rows whose maximum keeps growing); the raise rescales O in
// tensor memory and is warp-uniform because tcgen05 loads / stores are
// warp-collective.
template <bool kScaled, bool kSparse = false>
__device__ __forceinline__ void softmax_slot(const SoftmaxIo& io, uint32_t tmem, const Pair& pr, int warp, int lane,
                                             const WaitCtx& wc) {
  const int t = (warp - 4) >> 2;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + t * 128;
  const uint32_t tO = tmem + lane_base + 256 + t * 128;
  const uint32_t p_ready_even = cl(&io.p_ready[t], 0);
  const float c = io.scale_log2;
  const float rescale_gap = 15.0f / c;
  const int last_valid = io.N_kv - (io.n_kv - 1) * kTile;
  const int n = pr.row0[t] + row;
  float qs = 1.0f;
  if (kScaled && n < io.N) qs = __ldg(io.q_scale + n / 64);
  float m_used = 0.f, l = 0.f;
  bool ok = true;
  // the list is ascending, so the ragged last tile can only be its last entry
  const bool last_is_tail = !kSparse || (io.n_act > 0 && io.kv_list[io.n_act - 1] == io.n_kv - 1);
  for (int i = 0; i < io.n_act; ++i) {
    // key tile (read from the list only where the FP8 block scales need it)
    const int j = (kSparse && kScaled) ? static_cast<int>(io.kv_list[i]) : i;
    const bool tail_step = kSparse ? (i == io.n_act - 1 && last_is_tail) : (j == io.n_kv - 1);
    float sc0 = 1.0f, sc1 = 1.0f;
    if (kScaled) {
      const float ks0 = __ldg(io.k_scale + 2 * j);
      const float ks1 = 2 * j + 1 < io.n_blocks ? __ldg(io.k_scale + 2 * j + 1) : ks0;
      sc0 = qs * ks0;
      sc1 = qs * ks1;
    }
    if (!(ok = warp_wait(&io.s_full[t], i & 1, wc))) break;
    tc_fence_after();
    uint32_t s[128];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, s + q * 32);
    tmem_ld_wait128(s);
    float* f = reinterpret_cast<float*>(s);
    if (tail_step && last_valid < kTile) {            // keys past N in the last tile
#pragma unroll
      for (int e = 0; e < 128; ++e)
        if (e >= last_valid) f[e] = -INFINITY;
    }
    const float mx = kScaled ? fmaxf(max64(f) * sc0, max64(f + 64) * sc1) : max128(f);
    float alpha = 1.0f;
    bool rescale = false;
    if (i == 0) {
      m_used = mx;
    } else if (__any_sync(0xffffffffu, mx > m_used + rescale_gap)) {
      const float m_new = fmaxf(m_used, mx);
      alpha = ex2_approx((m_used - m_new) * c);
      m_used = m_new;
      l *= alpha;
      rescale = true;
    }
    const float neg = -m_used * c;
    float sum[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t pk[kSparse ? 16 : 32];
    if constexpr (kSparse) {
      // P in four stores of 16 columns: fewer live registers (the block-sparse
      // instance holds the tile list state as well); the same pairs, the
      // same order of the sums, the same bits as the dense instance
      static_assert(16 % kPolyEvery<kScaled> == 0, "the polynomial pairs must repeat every 16 pairs");
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        exp_pairs<16, kPolyEvery<kScaled>>(f + 32 * q, (kScaled && q >= 2) ? c * sc1 : (kScaled ? c * sc0 : c), neg,
                                           pk, sum);
        tmem_st16(tS + 16 * q, pk);
      }
    } else {
      exp_half<kPolyEvery<kScaled>>(f, kScaled ? c * sc0 : c, neg, pk, sum);
      tmem_st32(tS, pk);
      exp_half<kPolyEvery<kScaled>>(f + 64, kScaled ? c * sc1 : c, neg, pk, sum);
      tmem_st32(tS + 32, pk);
    }
    l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
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
    if (lane == 0) mbar_arrive_remote(p_ready_even);
  }
  // epilogue: O / l and the log-sum-exp (a row that sees no key tile: O = 0,
  // LSE = -inf, and tensor memory holds no product to read)
  if (ok && warp_wait(&io.o_final[t], 0, wc)) {
    tc_fence_after();
    const bool valid = n < io.N;
    const bool empty = kSparse && io.n_act == 0;
    const float inv_l = empty ? 0.f : __frcp_rn(l);   // reciprocal without the division slow-path call
    const size_t row_off = (static_cast<size_t>(pr.bh) * io.N + n) * kHeadDim;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t o[32];
      tmem_ld32(tO + q * 32, o);
      tmem_ld_wait(o);
      if (kSparse && empty) {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (valid) {
        if (io.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(io.out) + row_off + q * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                 __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(io.out) + row_off + q * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float* v8 = reinterpret_cast<const float*>(o + 8 * i);
            dst[i] = make_uint4(pack_bf16x2_rn(v8[0] * inv_l, v8[1] * inv_l),
                                pack_bf16x2_rn(v8[2] * inv_l, v8[3] * inv_l),
                                pack_bf16x2_rn(v8[4] * inv_l, v8[5] * inv_l),
                                pack_bf16x2_rn(v8[6] * inv_l, v8[7] * inv_l));
          }
        }
      }
    }
    if (valid && io.lse != nullptr) {
      io.lse[static_cast<size_t>(pr.bh) * io.N + n] =
          empty ? -INFINITY : (m_used * c + lg2_approx(l)) * 0.69314718055994530942f;
    }
  }
}


}  // namespace attn
}  // namespace dit
