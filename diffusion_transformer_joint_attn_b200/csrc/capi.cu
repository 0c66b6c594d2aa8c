// C-ABI entry points of libdit_attn: argument validation, status word and
// dispatch to the kernel launchers.  Declarations and contracts live in
// include/dit_attn.h.
#include <cstdint>
#include <mutex>

#include "dit_attn.h"
#include "launch.h"

namespace dit {

// The one static device allocation of the library: a status word that
// kernels set when a bounded wait gives up.  Its device address differs per
// device, so it is looked up with that device current and cached.
__device__ int g_status_word = 0;

int* device_status_word() {
  constexpr int kMaxDevices = 64;
  static int* cached[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<int*>(ptr);
  }
  return cached[dev];
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace dit

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// CUDA runtime error behind the last DIT_ERR_CUDA of this host thread.
thread_local int t_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DIT_OK;
  t_last_cuda_error = static_cast<int>(e);
  return DIT_ERR_CUDA;
}
// For launchers that return a dit_status_t: on DIT_ERR_CUDA take (and clear)
// the runtime's last error.
int launcher_status(int rc) {
  if (rc == DIT_ERR_CUDA) t_last_cuda_error = static_cast<int>(cudaGetLastError());
  return rc;
}

}  // namespace

extern "C" {

int dit_rope_table_build(const int32_t* pos, int N, int D, const int32_t* axes, double theta, float* rope_cos,
                         float* rope_sin, dit_stream_t stream) {
  if (pos == nullptr || axes == nullptr || rope_cos == nullptr || rope_sin == nullptr) return DIT_ERR_INVALID_ARG;
  if (N < 1 || !(theta > 0.0)) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if (axes[0] < 0 || axes[1] < 0 || axes[2] < 0 || (axes[0] | axes[1] | axes[2]) & 1 ||
      axes[0] + axes[1] + axes[2] != D)
    return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(N) * (D / 2) > (1LL << 40)) return DIT_ERR_INVALID_ARG;
  if (!aligned4(pos) || !aligned16(rope_cos) || !aligned16(rope_sin)) return DIT_ERR_MISALIGNED;
  dit::RopeTableArgs a{pos, N, D, {axes[0], axes[1], axes[2]}, theta, rope_cos, rope_sin};
  return cuda_status(dit::launch_rope_table(a, static_cast<cudaStream_t>(stream)));
}

int dit_rope_apply(const void* x, const float* rope_cos, const float* rope_sin, void* x_rot, int B, int H, int N,
                   int D, dit_stream_t stream) {
  if (x == nullptr || rope_cos == nullptr || rope_sin == nullptr || x_rot == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N > (1LL << 40)) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x_rot) || !aligned16(rope_cos) || !aligned16(rope_sin)) return DIT_ERR_MISALIGNED;
  dit::RopeApplyArgs a{x, rope_cos, rope_sin, x_rot, B, H, N, D};
  return cuda_status(dit::launch_rope_apply(a, static_cast<cudaStream_t>(stream)));
}

int dit_attn_prepare_kv(const void* k, const void* v, const float* rope_cos, const float* rope_sin, void* k_rot,
                        void* v_f16, int B, int H, int N, int D, dit_stream_t stream) {
  if (k == nullptr || v == nullptr || rope_cos == nullptr || rope_sin == nullptr || k_rot == nullptr ||
      v_f16 == nullptr)
    return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N > (1LL << 40)) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_rot) || !aligned16(v_f16) || !aligned16(rope_cos) ||
      !aligned16(rope_sin))
    return DIT_ERR_MISALIGNED;
  dit::PrepareKVArgs a{k, v, rope_cos, rope_sin, k_rot, v_f16, B, H, N, D};
  return cuda_status(dit::launch_prepare_kv(a, static_cast<cudaStream_t>(stream)));
}

int dit_attn_prepare_kv_split(const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                              void* k_split, void* v_f16, int B, int H, int N, int D, dit_stream_t stream) {
  if (k == nullptr || v == nullptr || k_split == nullptr || v_f16 == nullptr) return DIT_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N > (1LL << 40)) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_split) || !aligned16(v_f16)) return DIT_ERR_MISALIGNED;
  if (rope_cos != nullptr && (!aligned16(rope_cos) || !aligned16(rope_sin))) return DIT_ERR_MISALIGNED;
  dit::PrepareKVArgs a{k, v, rope_cos, rope_sin, k_split, v_f16, B, H, N, D};
  return cuda_status(dit::launch_prepare_kv_split(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Argument checks and launch shared by the dense, key-set and block-sparse
// entries: N_q queries attend to N_kv keys (N_q == N_kv except for
// dit_attn_forward_kv).  `kv_tables`: the rotary tables may be applied to k
// in the kernel (the keys are the query tokens).
int forward_bf16(const void* q, const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                 const uint8_t* kv_mask, void* out, float* lse, int B, int H, long long N_q, long long N_kv,
                 bool kv_tables, int D, int dtype, dit_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1) return DIT_ERR_INVALID_ARG;
  if (N_q < 1 || N_q > 0x7FFFFFFF || N_kv < 1 || N_kv > 0x7FFFFFFF) return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x3FFFFFFF) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  const bool split = (dtype & DIT_QK_SPLIT) != 0;
  if (split) {
    // the split form takes the prepared operands of dit_attn_prepare_kv_split
    if ((dtype & ~(DIT_OUT_F32 | DIT_QK_SPLIT | DIT_V_F16)) != DIT_BF16) return DIT_ERR_UNSUPPORTED;
    if (!(dtype & DIT_V_F16)) return DIT_ERR_INVALID_ARG;
    if (kv_mask != nullptr) return DIT_ERR_UNSUPPORTED;
  } else {
    if ((dtype & ~(DIT_OUT_F32 | DIT_K_ROTATED | DIT_V_F16)) != DIT_BF16) return DIT_ERR_UNSUPPORTED;
    if ((dtype & DIT_K_ROTATED) && rope_cos == nullptr) return DIT_ERR_INVALID_ARG;
    // tables for the queries only: k must come rotated
    if (!kv_tables && rope_cos != nullptr && !(dtype & DIT_K_ROTATED)) return DIT_ERR_INVALID_ARG;
  }
  if (kv_mask != nullptr && N_kv > static_cast<long long>(DIT_SPARSE_MAX_KV_TILES) * 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DIT_ERR_MISALIGNED;
  if ((rope_cos != nullptr && (!aligned16(rope_cos) || !aligned16(rope_sin))) || (lse != nullptr && !aligned4(lse)))
    return DIT_ERR_MISALIGNED;
  const bool out_f32 = (dtype & DIT_OUT_F32) != 0;
  if (split) {
    dit::AttnFwdSplitArgs a{q, k, v, rope_cos, rope_sin, out, lse, B, H, static_cast<int>(N_q), out_f32,
                            static_cast<int>(N_kv)};
    return launcher_status(dit::launch_attn_fwd_split(a, static_cast<cudaStream_t>(stream)));
  }
  dit::AttnFwdArgs a{q,
                     k,
                     v,
                     rope_cos,
                     rope_sin,
                     out,
                     lse,
                     B,
                     H,
                     static_cast<int>(N_q),
                     out_f32,
                     (dtype & DIT_K_ROTATED) != 0,
                     (dtype & DIT_V_F16) != 0,
                     kv_mask,
                     static_cast<int>(N_kv)};
  return launcher_status(dit::launch_attn_fwd_bf16(a, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int dit_attn_forward(const void* q, const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                     void* out, float* lse, int B, int H, int N_txt, int N_img, int D, int dtype,
                     dit_stream_t stream) {
  if (N_txt < 0 || N_img < 0) return DIT_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(N_txt) + N_img;
  return forward_bf16(q, k, v, rope_cos, rope_sin, nullptr, out, lse, B, H, N, N, true, D, dtype, stream);
}

int dit_attn_forward_kv(const void* q, const void* k, const void* v, const float* q_cos, const float* q_sin,
                        void* out, float* lse, int B, int H, int N_q, int N_kv, int D, int dtype,
                        dit_stream_t stream) {
  return forward_bf16(q, k, v, q_cos, q_sin, nullptr, out, lse, B, H, N_q, N_kv, false, D, dtype, stream);
}

size_t dit_attn_forward_host_workspace(int B, int H, int N, int D, int dtype, int chunk_heads) {
  if (B < 1 || H < 1 || N < 1 || chunk_heads < 1 || D != 128) return 0;
  if (static_cast<long long>(B) * H > 0x7FFFFFFF) return 0;
  if ((dtype & ~DIT_OUT_F32) != DIT_BF16) return 0;
  return dit::host_forward_workspace_bytes(B * H, N, chunk_heads, (dtype & DIT_OUT_F32) != 0);
}

}  // extern "C"

namespace {

// The argument checks of the host-buffer entries that need no workspace and
// no CUDA call.
int host_forward_args(const void* q, const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                      const void* out, int B, int H, int N_txt, int N_img, int D, int dtype, int chunk_heads) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N_txt < 0 || N_img < 0 || chunk_heads < 1) return DIT_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(N_txt) + N_img;
  if (N < 1 || N > 0x7FFFFFFF || static_cast<long long>(B) * H > 0x7FFFFFFF) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if ((dtype & ~DIT_OUT_F32) != DIT_BF16) return DIT_ERR_UNSUPPORTED;
  return DIT_OK;
}

}  // namespace

extern "C" {

int dit_attn_forward_host(const void* q, const void* k, const void* v, const float* rope_cos, const float* rope_sin,
                          void* out, float* lse, int B, int H, int N_txt, int N_img, int D, int dtype,
                          void* workspace, size_t workspace_bytes, int chunk_heads, dit_stream_t stream) {
  const int rc = host_forward_args(q, k, v, rope_cos, rope_sin, out, B, H, N_txt, N_img, D, dtype, chunk_heads);
  if (rc != DIT_OK) return rc;
  if (workspace == nullptr) return DIT_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(N_txt) + N_img;
  const bool out_f32 = (dtype & DIT_OUT_F32) != 0;
  if (workspace_bytes < dit::host_forward_workspace_bytes(B * H, static_cast<int>(N), chunk_heads, out_f32))
    return DIT_ERR_INVALID_ARG;
  if (!aligned16(workspace) || (rope_cos != nullptr && (!aligned16(rope_cos) || !aligned16(rope_sin))))
    return DIT_ERR_MISALIGNED;
  dit::HostForwardArgs a{q, k, v, rope_cos, rope_sin, out, lse, B, H, static_cast<int>(N), out_f32, workspace,
                         chunk_heads};
  return cuda_status(dit::host_forward(a, static_cast<cudaStream_t>(stream)));
}

int dit_attn_forward_host_static(const void* q, const void* k, const void* v, const float* rope_cos,
                                 const float* rope_sin, void* out, float* lse, int B, int H, int N_txt, int N_img,
                                 int D, int dtype, int chunk_heads, dit_stream_t stream) {
  // argument errors and an oversize problem are reported before any CUDA call
  int rc = host_forward_args(q, k, v, rope_cos, rope_sin, out, B, H, N_txt, N_img, D, dtype, chunk_heads);
  if (rc != DIT_OK) return rc;
  const long long N = static_cast<long long>(N_txt) + N_img;
  if (dit::host_forward_workspace_bytes(B * H, static_cast<int>(N), chunk_heads, (dtype & DIT_OUT_F32) != 0) >
      DIT_STATIC_WORKSPACE_BYTES)
    return DIT_ERR_WORKSPACE;
  void* ws = nullptr;
  rc = cuda_status(dit::static_workspace(&ws));
  if (rc != DIT_OK) return rc;
  return dit_attn_forward_host(q, k, v, rope_cos, rope_sin, out, lse, B, H, N_txt, N_img, D, dtype, ws,
                               DIT_STATIC_WORKSPACE_BYTES, chunk_heads, stream);
}

int dit_attn_forward_sparse(const void* q, const void* k, const void* v, const float* rope_cos,
                            const float* rope_sin, const uint8_t* kv_mask, void* out, float* lse, int B, int H,
                            int N_txt, int N_img, int D, int dtype, dit_stream_t stream) {
  if (kv_mask == nullptr) return DIT_ERR_INVALID_ARG;
  if (N_txt < 0 || N_img < 0) return DIT_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(N_txt) + N_img;
  return forward_bf16(q, k, v, rope_cos, rope_sin, kv_mask, out, lse, B, H, N, N, true, D, dtype, stream);
}

int dit_attn_quantize_fp8(const void* x_bf16, const float* rope_cos, const float* rope_sin, uint8_t* x_fp8,
                          float* scale, int B, int H, int N, int D, dit_stream_t stream) {
  if (x_bf16 == nullptr || x_fp8 == nullptr || scale == nullptr) return DIT_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * ((N + 63) / 64) > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(x_bf16) || !aligned16(x_fp8) || !aligned4(scale)) return DIT_ERR_MISALIGNED;
  if (rope_cos != nullptr && (!aligned16(rope_cos) || !aligned16(rope_sin))) return DIT_ERR_MISALIGNED;
  dit::QuantFp8Args a{x_bf16, rope_cos, rope_sin, x_fp8, scale, B, H, N};
  return cuda_status(dit::launch_quantize_fp8(a, static_cast<cudaStream_t>(stream)));
}

int dit_attn_forward_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* q_scale,
                         const float* k_scale, const float* v_scale, void* out, float* lse, int B, int H,
                         int N_txt, int N_img, int D, int dtype, dit_stream_t stream) {
  if (q8 == nullptr || k8 == nullptr || v8 == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (q_scale == nullptr || k_scale == nullptr || v_scale == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N_txt < 0 || N_img < 0) return DIT_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(N_txt) + N_img;
  if (N < 1 || N > 0x7FFFFFFF) return DIT_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7FFFFFFF) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if ((dtype & ~DIT_OUT_F32) != DIT_FP8_E4M3) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(out)) return DIT_ERR_MISALIGNED;
  if (!aligned4(q_scale) || !aligned4(k_scale) || !aligned4(v_scale) || (lse != nullptr && !aligned4(lse)))
    return DIT_ERR_MISALIGNED;
  dit::AttnFwdFp8Args a{q8, k8, v8, q_scale, k_scale, v_scale, out, lse, B, H, static_cast<int>(N),
                        (dtype & DIT_OUT_F32) != 0};
  return launcher_status(dit::launch_attn_fwd_fp8(a, static_cast<cudaStream_t>(stream)));
}

int dit_qkv_project_fp8(const void* x, const void* w, const float* bias, const float* rope_cos,
                        const float* rope_sin, uint8_t* q8, uint8_t* k8, uint8_t* v8, float* q_scale, float* k_scale,
                        float* v_scale, void* q16, void* k16, void* v16, int B, int N, int C, int H, int D,
                        dit_stream_t stream) {
  if (x == nullptr || w == nullptr || q8 == nullptr || k8 == nullptr || v8 == nullptr || q_scale == nullptr ||
      k_scale == nullptr || v_scale == nullptr)
    return DIT_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return DIT_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || C < 1 || H < 1) return DIT_ERR_INVALID_ARG;
  if (B > 65535 || static_cast<long long>(B) * H * N * 128 > (1LL << 40) || static_cast<long long>(C) * N * B > (1LL << 40))
    return DIT_ERR_INVALID_ARG;
  if (D != 128 || (H & 1) || (C & 7)) return DIT_ERR_UNSUPPORTED;
  const void* out16[3] = {q16, k16, v16};
  if (!aligned16(x) || !aligned16(w) || !aligned16(q8) || !aligned16(k8) || !aligned16(v8)) return DIT_ERR_MISALIGNED;
  if (!aligned4(q_scale) || !aligned4(k_scale) || !aligned4(v_scale) || (bias != nullptr && !aligned4(bias)))
    return DIT_ERR_MISALIGNED;
  if (rope_cos != nullptr && (!aligned16(rope_cos) || !aligned16(rope_sin))) return DIT_ERR_MISALIGNED;
  for (const void* o : out16)
    if (o != nullptr && !aligned16(o)) return DIT_ERR_MISALIGNED;
  dit::QkvProjArgs a{x,  w,  bias, rope_cos, rope_sin, {q8, k8, v8}, {q_scale, k_scale, v_scale},
                     {q16, k16, v16}, B, N, C, H};
  return launcher_status(dit::launch_qkv_proj_fp8(a, static_cast<cudaStream_t>(stream)));
}

static_assert(DIT_MERGE_MAX_PARTS == dit::kMergeMaxParts, "part limit of the header and the kernel differ");
static_assert(DIT_STATIC_WORKSPACE_BYTES == dit::kStaticWorkspaceBytes, "static workspace size differs");

int dit_attn_merge(const void* const* o_parts, const float* const* lse_parts, int R, void* out, float* lse_out,
                   int B, int H, int N, int D, int dtype, dit_stream_t stream) {
  if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (R < 1 || R > DIT_MERGE_MAX_PARTS) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return DIT_ERR_INVALID_ARG;
  if (D != 128) return DIT_ERR_UNSUPPORTED;
  if ((dtype & ~(DIT_PART_F32 | DIT_OUT_F32)) != DIT_BF16) return DIT_ERR_UNSUPPORTED;
  dit::MergeArgs a;
  for (int r = 0; r < R; ++r) {
    if (o_parts[r] == nullptr || lse_parts[r] == nullptr) return DIT_ERR_INVALID_ARG;
    if (!aligned16(o_parts[r]) || !aligned4(lse_parts[r])) return DIT_ERR_MISALIGNED;
    a.o[r] = o_parts[r];
    a.lse[r] = lse_parts[r];
  }
  if (!aligned16(out) || (lse_out != nullptr && !aligned4(lse_out))) return DIT_ERR_MISALIGNED;
  a.R = R;
  a.out = out;
  a.lse_out = lse_out;
  a.rows = static_cast<long long>(B) * H * N;
  a.in_f32 = (dtype & DIT_PART_F32) != 0;
  a.out_f32 = (dtype & DIT_OUT_F32) != 0;
  return cuda_status(dit::launch_merge(a, static_cast<cudaStream_t>(stream)));
}

int dit_attn_wait_selftest(long long limit_ns, dit_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000LL) return DIT_ERR_INVALID_ARG;
  return cuda_status(dit::launch_wait_selftest(static_cast<unsigned long long>(limit_ns),
                                               static_cast<cudaStream_t>(stream)));
}

int dit_attn_get_status(int* status_host, dit_stream_t stream) {
  if (status_host == nullptr) return DIT_ERR_INVALID_ARG;
  int* word = dit::device_status_word();
  if (word == nullptr) return DIT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int value = 0;
  int rc = cuda_status(cudaMemcpyAsync(&value, word, sizeof(int), cudaMemcpyDeviceToHost, s));
  if (rc == DIT_OK) rc = cuda_status(cudaMemsetAsync(word, 0, sizeof(int), s));
  if (rc == DIT_OK) rc = cuda_status(cudaStreamSynchronize(s));
  if (rc != DIT_OK) return rc;
  *status_host = value;
  return DIT_OK;
}

int dit_attn_last_cuda_error(void) { return t_last_cuda_error; }

const char* dit_attn_last_cuda_error_string(void) {
  return cudaGetErrorString(static_cast<cudaError_t>(t_last_cuda_error));
}

const char* dit_attn_status_string(int status) {
  switch (status) {
    case DIT_OK: return "ok";
    case DIT_ERR_INVALID_ARG: return "invalid argument";
    case DIT_ERR_UNSUPPORTED: return "unsupported head dimension, dtype or flag";
    case DIT_ERR_MISALIGNED: return "pointer not aligned (16 bytes; 4 for lse)";
    case DIT_ERR_CUDA: return "CUDA runtime or driver call failed";
    case DIT_ERR_TIMEOUT: return "a device-side wait timed out";
    case DIT_ERR_WORKSPACE: return "problem needs more workspace than the static workspace holds";
    default: return "unknown status";
  }
}

}  // extern "C"
