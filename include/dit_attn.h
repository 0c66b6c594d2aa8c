/*
 * dit_attn.h — C ABI of libdit_attn: joint text+image attention for
 * FLUX-style diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * What it computes.  Inside every DiT block the text tokens, the noisy
 * target-image tokens and (for image-to-image) the reference-image tokens are
 * concatenated and attend to each other in one shared, bidirectional attention
 * layer (bpdata.com "FLUX 3 Image Klein optimalizálása", section "Modellezés
 * és pipeline jellemzők").  Plain BF16 attention is about 60 % of the DiT's
 * GPU kernel time at 2048x2048 (scopeai.cc FLUX 3 Klein story, section on the
 * effect of each optimisation).  For each batch item b and head h:
 *
 *     q~_n = R(pos_n) q_n,  k~_m = R(pos_m) k_m      three-axis rotary embedding
 *     O_n  = sum_m softmax_m(q~_n . k~_m / sqrt(D)) v_m
 *     LSE_n = ln sum_m exp(q~_n . k~_m / sqrt(D))
 *
 * R(pos) turns channel pair (2j, 2j+1) by the angle pos_a * theta^(-2i/d_a),
 * where axis a in (t, h, w) owns the consecutive channel slice of width d_a
 * that contains the pair and i is the pair's index inside that slice.
 *
 * Conventions shared by every entry point:
 *   - Layout: q, k, v, out are [B][H][N][D] row-major, N = N_txt + N_img
 *     tokens in sequence order [text | image(s)]; lse is [B][H][N].
 *   - Ownership: the caller allocates and owns every buffer.  The library
 *     allocates no device memory per call; its device image holds one status
 *     word and the DIT_STATIC_WORKSPACE_BYTES array of
 *     dit_attn_forward_host_static.  Inputs are only read; outputs are fully
 *     overwritten.
 *   - Streams: every call is asynchronous on `stream` (a cudaStream_t, NULL =
 *     legacy default stream) and does not synchronise the host, except
 *     dit_attn_get_status.
 *   - Errors: every call returns a dit_status_t.  Argument errors are found on
 *     the host before anything is launched.  A device-side wait that exceeds
 *     its time limit makes the kernel exit early and records DIT_ERR_TIMEOUT
 *     in the status word, read by dit_attn_get_status.
 */
#ifndef DIT_ATTN_H
#define DIT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* dit_stream_t; /* a cudaStream_t */

typedef enum {
  DIT_OK = 0,
  DIT_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, sizes that overflow */
  DIT_ERR_UNSUPPORTED = -2, /* D != 128, unknown dtype or flag */
  DIT_ERR_MISALIGNED = -3,  /* a pointer is not 16-byte aligned (4-byte for lse) */
  DIT_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed (launch, tensor map) */
  DIT_ERR_TIMEOUT = -5,     /* a device-side wait gave up (read via dit_attn_get_status) */
  DIT_ERR_WORKSPACE = -6    /* dit_attn_forward_host_static: the problem needs more than the static workspace */
} dit_status_t;

/* Element type of q/k/v, OR-able with the flags below. */
typedef enum { DIT_BF16 = 0, DIT_FP8_E4M3 = 1 } dit_dtype_t;
#define DIT_OUT_F32 0x100   /* write `out` as fp32 instead of bf16 */
#define DIT_K_ROTATED 0x200 /* k already carries the rotary embedding (dit_rope_apply); rotate q only */
#define DIT_V_F16 0x400     /* v is given as fp16 (dit_attn_prepare_kv) instead of bf16 */
#define DIT_PART_F32 0x800  /* dit_attn_merge: the part outputs are fp32 instead of bf16 */
#define DIT_QK_SPLIT 0x1000 /* compensated q~ k~^T on fp16 hi + lo operands (dit_attn_prepare_kv_split) */
#define DIT_SPARSE_MAX_KV_TILES 4096  /* dit_attn_forward_sparse: N <= 4096 x 128 keys */
#define DIT_MERGE_MAX_PARTS 16

/*
 * dit_rope_table_build — cos/sin table of the three-axis rotary embedding.
 *
 *   pos       device int32 [N][3]: (t, h, w) position of every token.  In the
 *             FLUX joint sequence text tokens sit at (0,0,0), target-image
 *             latent pixel (row, col) at (0,row,col) and a reference image's at
 *             (1,row,col).
 *   N         number of tokens, >= 1.
 *   D         head dimension, 128.
 *   axes      HOST int32[3]: channels per axis (t, h, w), each even, sum == D,
 *             e.g. {16, 56, 56}; slices are consecutive in that order.
 *   theta     frequency base, > 0 (10000 for FLUX).
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2], written: entry [n][j] is cos/sin of the
 *             angle of channel pair (2j, 2j+1) at token n,
 *             pos[n][a] * theta^(-2i/d_a) with (a, i) the pair's axis and
 *             index inside that axis; evaluated in fp64, rounded to fp32.
 * Pointers 16-byte aligned.  Runs once per resolution, not per attention call.
 */
int dit_rope_table_build(const int32_t* pos, int N, int D, const int32_t* axes, double theta, float* rope_cos,
                         float* rope_sin, dit_stream_t stream);

/*
 * dit_rope_apply — x_rot = R(pos) x for bf16 x [B][H][N][D] (the rotation of
 * dit_attn_forward, as a separate memory-bound pass).
 *
 *   x         device bf16 [B][H][N][D].
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2] from dit_rope_table_build.
 *   x_rot     device bf16 [B][H][N][D], written; may equal x (in place).
 *   B, H, N   >= 1;  D must be 128.
 * Each rotated component is the bf16 nearest (ties to even) to the exact
 * value x_2j*cos - x_2j+1*sin (resp. x_2j*sin + x_2j+1*cos) of the fp32 table
 * entries, so dit_attn_forward(q, dit_rope_apply(k), ..., DIT_K_ROTATED)
 * returns bit-for-bit what dit_attn_forward(q, k, ...) does.  Rotating K
 * once here instead of once per query tile inside the attention kernel is the
 * faster composition for long sequences.  All pointers 16-byte aligned.
 */
int dit_rope_apply(const void* x, const float* rope_cos, const float* rope_sin, void* x_rot, int B, int H, int N,
                   int D, dit_stream_t stream);

/*
 * dit_attn_prepare_kv — the operands of the attention's two products,
 * prepared once per call in one memory-bound pass:
 *
 *   k, v      device bf16 [B][H][N][D].
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2] from dit_rope_table_build.
 *   k_rot     device bf16 [B][H][N][D], written: k rotated exactly as by
 *             dit_rope_apply.
 *   v_f16     device fp16 [B][H][N][D], written: v converted to fp16 (exact for
 *             2^-14 <= |v| <= 65504; |v| > 65504 is outside the contract).
 *   B, H, N   >= 1;  D must be 128.  All pointers 16-byte aligned.
 * dit_attn_forward(q, k_rot, v_f16, ..., DIT_K_ROTATED | DIT_V_F16) returns bit
 * for bit what dit_attn_forward(q, k, v, ...) does, and is the fast path: the
 * attention kernel then does no per-tile operand work for K and V.
 */
int dit_attn_prepare_kv(const void* k, const void* v, const float* rope_cos, const float* rope_sin, void* k_rot,
                        void* v_f16, int B, int H, int N, int D, dit_stream_t stream);

/*
 * dit_attn_prepare_kv_split — the operands of the split (compensated) form of
 * the attention, DIT_QK_SPLIT, prepared once per call in one memory-bound
 * pass.  That form exists for inputs whose logits are so large that one bf16
 * rounding of the rotated q and k visibly moves the output: with activation
 * outliers (channels x16, as modelled for the 2048x2048 workloads) the logits
 * have a standard deviation of ~45, and the bf16 operand rounding alone moves
 * O by up to ~7 against exact attention.  The split form keeps such outputs
 * within the library's BF16 parity bar (max-abs 2e-2, mean-abs 2e-3 against
 * fp64 attention of the same inputs).
 *
 *   k, v      device bf16 [B][H][N][D].
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2] from dit_rope_table_build, or both NULL
 *             (no rotary embedding).
 *   k_split   device fp16 [2][B][H][N][D], written: plane 0 holds hi, plane 1
 *             lo, of r = RN32(RN64(rotated k component)) (both table products
 *             are exact in fp64): hi = the fp16 nearest r, lo = the fp16
 *             nearest r - hi, so hi + lo = r to within 2^-22 |r| (2^-25
 *             absolute where lo is subnormal).  |r| must stay below 65504.
 *   v_f16     device fp16 [B][H][N][D], written: fp16(v) as dit_attn_prepare_kv.
 *   B, H, N   >= 1;  D must be 128.  All pointers 16-byte aligned.
 */
int dit_attn_prepare_kv_split(const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                              void* k_split, void* v_f16, int B, int H, int N, int D, dit_stream_t stream);

/*
 * dit_attn_forward — joint attention forward, BF16 in, BF16 (or fp32) out.
 *
 *   q, k, v   device bf16 [B][H][N][D], N = N_txt + N_img.
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2] from dit_rope_table_build, applied to q and
 *             k inside the kernel; both NULL = no rotary embedding.
 *   out       device [B][H][N][D], bf16, or fp32 when dtype has DIT_OUT_F32.
 *   lse       device fp32 [B][H][N] or NULL: natural-log log-sum-exp of the
 *             scaled logits q~.k~/sqrt(D) of every query row.
 *   B, H      batch (e.g. 2 for the two classifier-free-guidance branches) and
 *             heads, >= 1.
 *   N_txt, N_img
 *             text and image token counts, >= 0, N_txt + N_img >= 1.  Every
 *             token attends to all N tokens (no mask); positions enter only
 *             through the tables.
 *   D         head dimension; must be 128.
 *   dtype     DIT_BF16, optionally | DIT_OUT_F32, | DIT_K_ROTATED (requires
 *             the tables: they are then applied to q only) and | DIT_V_F16
 *             (v holds fp16 values, as written by dit_attn_prepare_kv).
 *             Or the split form: DIT_BF16 | DIT_QK_SPLIT | DIT_V_F16
 *             [| DIT_OUT_F32], with k the fp16 [2][B][H][N][D] operand and v
 *             the fp16 values of dit_attn_prepare_kv_split (made with the same
 *             tables, or none).  The kernel rotates q as that call rotates k,
 *             splits it into fp16 hi + lo and accumulates
 *             q~ k~^T = hi_q.lo_k + lo_q.hi_k + hi_q.hi_k in fp32: the logits
 *             carry ~2^-21 relative error instead of a bf16 operand's 2^-8,
 *             at three times the tensor-core work of q k^T.
 *
 * Precision: each rotated component of q and k is the bf16 nearest to its
 * exact value for the fp32 table entries; q~ k~^T accumulates in fp32; the
 * softmax runs in fp32; P (in [0, 2^15]) and v are fp16 tensor-core operands
 * (v must satisfy |v| <= 65504; the bf16 -> fp16 conversion of v is exact for
 * |v| >= 2^-14), P v accumulates in fp32.
 * All pointers 16-byte aligned except lse (4-byte).  One kernel launch, no
 * host synchronisation, no allocation.  The first call on a device also sets
 * the kernel's shared-memory limit and looks up the status word's address;
 * make it outside any stream capture (capture of later calls is not tested).
 */
int dit_attn_forward(const void* q, const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                     void* out, float* lse, int B, int H, int N_txt, int N_img, int D, int dtype,
                     dit_stream_t stream);

/*
 * dit_attn_forward_kv — dit_attn_forward of N_q queries against a separate
 * set of N_kv keys and values: one part of key-sharded (context-parallel)
 * attention, where each part's (out, lse) covers a disjoint key set and
 * dit_attn_merge combines the parts into the attention over all keys
 * (wavespeed.ai "Beschleunigung der FLUX.1-dev Bildgenerierung", section on
 * context parallelism and First Block Cache).
 *
 *   q         device bf16 [B][H][N_q][D].
 *   k, v      device [B][H][N_kv][D] (k bf16, or the fp16 [2][B][H][N_kv][D]
 *             split operand with DIT_QK_SPLIT; v bf16, or fp16 with DIT_V_F16).
 *   q_cos, q_sin
 *             device fp32 [N_q][D/2]: the rotary table rows of the QUERY
 *             tokens (a contiguous slice of the full table when the queries
 *             are a contiguous token range), or both NULL.  The kernel rotates
 *             only q: with tables, k must come rotated (DIT_K_ROTATED, from
 *             dit_attn_prepare_kv / dit_rope_apply with the key tokens' rows)
 *             or split (DIT_QK_SPLIT, from dit_attn_prepare_kv_split).
 *   out, lse  device [B][H][N_q][D] and fp32 [B][H][N_q] (lse may be NULL):
 *             softmax over the N_kv keys only, and its log-sum-exp.
 *   N_q, N_kv >= 1.
 *   dtype     as dit_attn_forward; DIT_K_ROTATED is required when tables are
 *             given without DIT_QK_SPLIT.
 * With N_q == N_kv, the same tokens and tables, it returns bit for bit what
 * dit_attn_forward does.  Same limits, alignment and status handling.
 */
int dit_attn_forward_kv(const void* q, const void* k, const void* v, const float* q_cos, const float* q_sin,
                        void* out, float* lse, int B, int H, int N_q, int N_kv, int D, int dtype,
                        dit_stream_t stream);

/*
 * dit_attn_forward_host — dit_attn_forward on q, k, v in HOST memory, with
 * the results written to host memory: the library moves chunks of
 * chunk_heads (b, h) pairs through `workspace`, overlapping the copies to the
 * device, the kernels (K rotation and V conversion, then the forward) and the
 * copies back for consecutive chunks.  With page-locked host buffers the call
 * takes about as long as the larger of its two copy directions; pageable
 * buffers work but copy synchronously.
 *
 *   q, k, v     host bf16 [B][H][N][D].  They are read asynchronously: keep
 *               them unchanged until `stream` has been synchronised.
 *   rope_cos, rope_sin
 *               DEVICE fp32 [N][D/2] tables (dit_rope_table_build), or both
 *               NULL for no rotary embedding.
 *   out, lse    host [B][H][N][D] bf16 (fp32 with DIT_OUT_F32) and fp32
 *               [B][H][N] (lse may be NULL); complete once `stream` has been
 *               synchronised.
 *   dtype       DIT_BF16, optionally | DIT_OUT_F32.
 *   workspace   device memory of at least
 *               dit_attn_forward_host_workspace(B, H, N, D, dtype,
 *               chunk_heads) bytes, 16-byte aligned; owned by the caller.
 *               Consecutive calls may share it (the library orders its
 *               reuse); concurrent calls must not.
 *   chunk_heads at most this many (b, h) pairs per chunk, >= 1; the first
 *               and the last chunk hold one pair, so that little is left
 *               unoverlapped at either end.
 * The kernels run on `stream`; the copies on two streams the library creates
 * once per device, ordered after the work already queued on `stream`, and
 * `stream` waits for the last copy back.  Same limits and status handling as
 * dit_attn_forward; a workspace smaller than required is
 * DIT_ERR_INVALID_ARG.
 */
size_t dit_attn_forward_host_workspace(int B, int H, int N, int D, int dtype, int chunk_heads);
int dit_attn_forward_host(const void* q, const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                          void* out, float* lse, int B, int H, int N_txt, int N_img, int D, int dtype,
                          void* workspace, size_t workspace_bytes, int chunk_heads, dit_stream_t stream);

/*
 * dit_attn_forward_host_static — dit_attn_forward_host without a caller
 * workspace: the library uses a device array of DIT_STATIC_WORKSPACE_BYTES
 * that is part of its own device image, so the call allocates nothing.  It
 * is meant for callers that cannot hand the library device memory of their
 * own: code whose device memory is all owned by another runtime's pool or a
 * fixed budget, or latency-critical loops in which an allocation (which may
 * synchronise the device) is not acceptable.  The pages describe no such
 * entry point; it has no counterpart there.
 *
 * Arguments, results and status handling as dit_attn_forward_host, minus the
 * workspace.  When dit_attn_forward_host_workspace(B, H, N, D, dtype,
 * chunk_heads) exceeds DIT_STATIC_WORKSPACE_BYTES the call returns
 * DIT_ERR_WORKSPACE and does nothing.  Fewer heads per chunk need less, but
 * each of the three chunk buffers holds at least one head (about 1540 N bytes
 * with bf16 output, 1796 N with fp32), so whatever chunk_heads is, only
 * N <= DIT_STATIC_MAX_N_BF16_OUT (7262) tokens fit with bf16 output and
 * N <= DIT_STATIC_MAX_N_F32_OUT (6227) with fp32 output: a 1024x1024 image
 * (N = 4608) fits, the 2048x2048 (N = 16896) and image-to-image shapes do not.
 * Every call on a device uses the same array: calls that could overlap (from
 * several host threads, or on streams not ordered with each other) race on
 * it and must be serialised by the caller.  The first call on each device
 * looks the array's address up (and creates the copy streams); make that
 * first call outside any stream capture.
 */
#define DIT_STATIC_WORKSPACE_BYTES (32u << 20)
#define DIT_STATIC_MAX_N_BF16_OUT 7262
#define DIT_STATIC_MAX_N_F32_OUT 6227
int dit_attn_forward_host_static(const void* q, const void* k, const void* v, const float* rope_cos,
                                 const float* rope_sin, void* out, float* lse, int B, int H, int N_txt, int N_img,
                                 int D, int dtype, int chunk_heads, dit_stream_t stream);

/*
 * dit_attn_forward_sparse — dit_attn_forward restricted to the key tiles a
 * block mask selects, skipping the others entirely (no load, no product, no
 * exponential).  The pages name sparse attention only as prior art
 * (Sol-Attention and VC-Attention on B200: scopeai.cc, section on the effect
 * of each optimisation) and give no rule for choosing tiles, so the mask is an
 * input.
 *
 *   kv_mask   device uint8 [B][H][ceil(N/512)][ceil(N/128)]: query row n of
 *             (b, h) attends to key m only where
 *             kv_mask[b][h][n / 512][m / 128] is nonzero (512-row query
 *             blocks x 128-key tiles, the kernel's units of work).  A row
 *             whose block selects no tile gets out = 0 and lse = -inf (the
 *             sum over an empty key set), which dit_attn_merge treats as an
 *             empty part.
 *   N         at most DIT_SPARSE_MAX_KV_TILES x 128, else
 *             DIT_ERR_UNSUPPORTED.
 * Everything else (arguments, dtype flags, alignment, status) as
 * dit_attn_forward; an all-ones mask gives dit_attn_forward's result bit for
 * bit.
 */
int dit_attn_forward_sparse(const void* q, const void* k, const void* v, const float* rope_cos,
                            const float* rope_sin, const uint8_t* kv_mask, void* out, float* lse, int B, int H,
                            int N_txt, int N_img, int D, int dtype, dit_stream_t stream);

/*
 * dit_attn_quantize_fp8 — FP8 E4M3 operands for dit_attn_forward_fp8.
 *
 *   x_bf16    device bf16 [B][H][N][D] (q, k or v).
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2]: rotate first (q and k), or both NULL (v).
 *             Each rotated value x c - y s (or x s + y c) is evaluated in
 *             fp64 from the fp32 table entries (both products exact, one
 *             rounding of the sum) and then rounded to fp32.
 *   x_fp8     device uint8 [B][H][N][D], written: E4M3 ("e4m3fn": bias 7,
 *             largest finite 448, no infinities) codes.
 *   scale     device fp32 [B][H][ceil(N/64)], written: one scale per block of
 *             64 consecutive tokens x all D channels of one (b, h):
 *             amax / 448 in fp32, or 1 for an all-zero block.
 *   B, H, N   >= 1;  D must be 128.
 * Each element's code is the E4M3 value nearest (ties to even) to the fp32
 * quotient x / scale, saturated to +-448; x = code * scale approximately.
 * x_bf16, x_fp8 and the tables 16-byte aligned, scale 4-byte aligned.
 * FP8 attention is prior art on the pages (cuDNN FP8, VC-Attention FP8 on
 * B200: scopeai.cc, section on each optimisation's effect); the block scheme
 * is this library's.
 */
int dit_attn_quantize_fp8(const void* x_bf16, const float* rope_cos, const float* rope_sin, uint8_t* x_fp8,
                          float* scale, int B, int H, int N, int D, dit_stream_t stream);

/*
 * dit_attn_forward_fp8 — joint attention on FP8 E4M3 operands (dit_attn_quantize_fp8
 * output; the rotary embedding of q and k was applied before quantisation).
 *
 *   q8, k8, v8  device uint8 [B][H][N][D] E4M3 codes, N = N_txt + N_img.
 *   q_scale, k_scale, v_scale
 *               device fp32 [B][H][ceil(N/64)]: the value of a code in
 *               token block n/64 is code * scale.
 *   out         device [B][H][N][D], bf16, or fp32 when dtype has DIT_OUT_F32.
 *   lse         device fp32 [B][H][N] or NULL: natural-log sum-exp of the
 *               scaled logits of each row.
 *   dtype       DIT_FP8_E4M3, optionally | DIT_OUT_F32.
 * Computes softmax(q k^T / sqrt(D)) v of the dequantised values: S is formed
 * from the codes on the 8-bit tensor cores and scaled per (query block, key
 * block) in fp32; P (fp16) multiplies v dequantised to fp16 (code * scale,
 * rounded once), accumulating in fp32.  Same limits, alignment (16 bytes for
 * every pointer, 4 for the scales and lse), status words and asynchrony as
 * dit_attn_forward.
 */
int dit_attn_forward_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* q_scale,
                         const float* k_scale, const float* v_scale, void* out, float* lse, int B, int H,
                         int N_txt, int N_img, int D, int dtype, dit_stream_t stream);

/*
 * dit_qkv_project_fp8 — the QKV projection of the joint token sequence with
 * the FP8 operands of dit_attn_forward_fp8 made in the GEMM's epilogue
 * (the pages list GEMMs with epilogue fusion among the optimisations of
 * FLUX 3 Klein on B200: bpdata.com "FLUX 3 Image Klein optimalizálása",
 * sections on what the optimisation includes and on the detailed steps):
 *
 *     y[b][n][o] = sum_c x[b][n][c] w[o][c] (+ bias[o]),   o = s*H*D + h*D + d
 *
 * for s = 0, 1, 2 (q, k, v), accumulated in fp32 on the tensor cores, then,
 * per (s, b, h) without writing y to memory: q and k rotated exactly as by
 * dit_attn_quantize_fp8 (each pair turned in fp64 from the fp32 y and the fp32
 * table entries, rounded to fp32), and every block of 64 tokens x D channels
 * quantised as by dit_attn_quantize_fp8 (scale = amax / 448 in fp32, 1 for an
 * all-zero block; codes = E4M3 of y / scale, nearest even, saturating).
 *
 *   x         device bf16 [B][N][C]: hidden states of the joint sequence.
 *   w         device bf16 [3 H D][C]: the projection weight (rows: q heads,
 *             then k heads, then v heads; row-major like a linear layer).
 *   bias      device fp32 [3 H D] or NULL.
 *   rope_cos, rope_sin
 *             device fp32 [N][D/2] (dit_rope_table_build) or both NULL.
 *   q8, k8, v8
 *             device uint8 [B][H][N][D], written: E4M3 codes.
 *   q_scale, k_scale, v_scale
 *             device fp32 [B][H][ceil(N/64)], written.
 *   q16, k16, v16
 *             device bf16 [B][H][N][D] or NULL: the unrotated projection
 *             rounded to bf16 (the inputs of the BF16 path), written if given.
 *   B, N      >= 1.  C >= 1 with C % 8 == 0.  H >= 1 and even (256 output
 *             features per tile).  D must be 128.
 * Pointers 16-byte aligned except bias and the scales (4-byte).  Because the
 * sums are formed in fp32 in the tensor cores' order, a code can differ by
 * one step from the code of the exact projection where y / scale lies
 * within the accumulation error of a rounding midpoint.
 */
int dit_qkv_project_fp8(const void* x, const void* w, const float* bias, const float* rope_cos,
                        const float* rope_sin, uint8_t* q8, uint8_t* k8, uint8_t* v8, float* q_scale, float* k_scale,
                        float* v_scale, void* q16, void* k16, void* v16, int B, int N, int C, int H, int D,
                        dit_stream_t stream);

/*
 * dit_attn_merge — combine R partial results of the same queries over
 * disjoint key sets into the result over their union (context parallelism:
 * wavespeed.ai "Beschleunigung der FLUX.1-dev Bildgenerierung", section on
 * context parallelism and First Block Cache):
 *     lse = ln sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) O_r.
 *
 *   o_parts   HOST array of R device pointers, each [B][H][N][D] bf16 (fp32
 *             with DIT_PART_F32): the normalised partial outputs, as
 *             dit_attn_forward writes them.
 *   lse_parts HOST array of R device pointers, each [B][H][N] fp32.  A part
 *             with lse = -inf has no keys: its weight is 0 and the values of
 *             its output row are not used (they may be NaN; the memory must
 *             still be readable).
 *   R         1 .. DIT_MERGE_MAX_PARTS.
 *   out       device [B][H][N][D], bf16 (fp32 with DIT_OUT_F32).  Rows whose
 *             parts are all empty get 0.  May be the same buffer as one of
 *             the parts (same dtype): each element is read before written.
 *   lse_out   device fp32 [B][H][N] or NULL; may be one of lse_parts.
 *   dtype     DIT_BF16, optionally | DIT_PART_F32 | DIT_OUT_F32.
 * The parts may be in another GPU's memory if that memory is accessible from
 * the current device (peer access enabled or an imported IPC mapping): the
 * kernel reads them with ordinary loads.  Weights use expf / logf in fp32.
 * Alignment: parts and out 16 bytes, lse arrays 4 bytes.  D must be 128.
 */
int dit_attn_merge(const void* const* o_parts, const float* const* lse_parts, int R, void* out, float* lse_out,
                   int B, int H, int N, int D, int dtype, dit_stream_t stream);

/*
 * dit_attn_wait_selftest — exercise the bounded device-side waits that every
 * kernel of the library uses: a one-thread kernel waits for a barrier phase
 * that nothing completes, gives up after limit_ns nanoseconds
 * (1 us .. 1 s), records DIT_ERR_TIMEOUT in the status word and returns.
 * dit_attn_get_status then reports (and clears) DIT_ERR_TIMEOUT; the CUDA
 * context stays usable.  Returns DIT_OK once launched, DIT_ERR_INVALID_ARG
 * for a limit outside the range.
 */
int dit_attn_wait_selftest(long long limit_ns, dit_stream_t stream);

/*
 * dit_attn_get_status — synchronise `stream`, copy the device status word to
 * *status_host (DIT_OK or DIT_ERR_TIMEOUT) and reset it to DIT_OK.  Returns
 * DIT_OK, or DIT_ERR_CUDA if the synchronisation or copy failed (for example
 * after a device fault), or DIT_ERR_INVALID_ARG for a NULL status_host.
 */
int dit_attn_get_status(int* status_host, dit_stream_t stream);

/*
 * dit_attn_last_cuda_error — the CUDA runtime error code (a cudaError_t)
 * behind the most recent DIT_ERR_CUDA returned to this host thread, or 0 if
 * there was none or the failing call was a driver call that leaves no runtime
 * error (the tensor-map encoding).  dit_attn_last_cuda_error_string gives the
 * runtime's description of that code.  Neither makes a CUDA call that can
 * fail; both may be called without a GPU.
 */
int dit_attn_last_cuda_error(void);
const char* dit_attn_last_cuda_error_string(void);

/* Static English description of a dit_status_t value. */
const char* dit_attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* DIT_ATTN_H */
