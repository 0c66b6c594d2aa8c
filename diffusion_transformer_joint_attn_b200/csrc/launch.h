// Host-side launchers shared between the C-ABI shim and the kernel files.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace dit {

// Device status word of the current device (see capi.cu).
int* device_status_word();

struct RopeTableArgs {
  const int32_t* pos;
  int N;
  int D;
  int axes[3];
  double theta;
  float* cos;
  float* sin;
};
cudaError_t launch_rope_table(const RopeTableArgs& a, cudaStream_t s);

struct RopeApplyArgs {
  const void* x;
  const float* cos;
  const float* sin;
  void* y;
  int B, H, N, D;
};
cudaError_t launch_rope_apply(const RopeApplyArgs& a, cudaStream_t s);

struct PrepareKVArgs {
  const void* k;
  const void* v;
  const float* cos;
  const float* sin;
  void* k_rot;     // bf16, rotated
  void* v_f16;     // fp16 copy of v
  int B, H, N, D;
};
cudaError_t launch_prepare_kv(const PrepareKVArgs& a, cudaStream_t s);
// Same arguments; k_rot receives the fp16 split operand [2][B][H][N][D] (hi,
// then lo) and the tables may be null (no rotation).
cudaError_t launch_prepare_kv_split(const PrepareKVArgs& a, cudaStream_t s);

struct QuantFp8Args {
  const void* x;       // bf16 [B][H][N][128]
  const float* cos;    // [N][64] or nullptr (no rotation)
  const float* sin;
  void* codes;         // e4m3 [B][H][N][128]
  float* scale;        // [B][H][ceil(N/64)]
  int B, H, N;
};
cudaError_t launch_quantize_fp8(const QuantFp8Args& a, cudaStream_t s);

struct AttnFwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* cos;
  const float* sin;
  void* out;
  float* lse;
  int B, H, N;
  bool out_f32;
  bool k_rotated;   // k already carries the rotary embedding: rotate q only
  bool v_f16;       // v is given as fp16 (otherwise bf16)
  const uint8_t* kv_mask = nullptr;   // [B*H][ceil(N/512)][ceil(N_kv/128)] block mask, or nullptr (dense)
  int N_kv = 0;     // keys per (b, h) of k and v; 0: N (queries and keys are the same tokens)
};
struct AttnFwdFp8Args {
  const void* q8;      // e4m3 [B][H][N][128]
  const void* k8;
  const void* v8;
  const float* q_scale;   // [B][H][ceil(N/64)]
  const float* k_scale;
  const float* v_scale;
  void* out;
  float* lse;
  int B, H, N;
  bool out_f32;
};
int launch_attn_fwd_fp8(const AttnFwdFp8Args& a, cudaStream_t s);

constexpr int kMergeMaxParts = 16;
struct MergeArgs {
  const void* o[kMergeMaxParts];      // part outputs [rows][128], bf16 or fp32
  const float* lse[kMergeMaxParts];   // part log-sum-exps [rows]
  int R;
  void* out;
  float* lse_out;                     // may be null
  long long rows;
  bool in_f32, out_f32;
};
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s);

// Host-buffer forward (host_pipeline.cu): q, k, v, out, lse in host memory,
// moved through `workspace` in chunks of chunk_heads (b, h) pairs.
struct HostForwardArgs {
  const void* q;       // host bf16 [B][H][N][128]
  const void* k;
  const void* v;
  const float* cos;    // device tables [N][64] or nullptr
  const float* sin;
  void* out;           // host bf16 (fp32 if out_f32)
  float* lse;          // host fp32 [B][H][N] or nullptr
  int B, H, N;
  bool out_f32;
  void* workspace;     // device, host_forward_workspace_bytes(...)
  int chunk_heads;
};
size_t host_forward_workspace_bytes(int BH, int N, int chunk_heads, bool out_f32);
// The library's static workspace for dit_attn_forward_host_static: its device
// address on the current device (looked up once per device).
constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;
cudaError_t static_workspace(void** out);
cudaError_t host_forward(const HostForwardArgs& a, cudaStream_t s);

// QKV projection with the FP8 operand epilogue (qkv_proj.cu).
struct QkvProjArgs {
  const void* x;         // bf16 [B][N][C]
  const void* w;         // bf16 [3 H 128][C]
  const float* bias;     // [3 H 128] or nullptr
  const float* cos;      // [N][64] or nullptr (no rotary embedding)
  const float* sin;
  uint8_t* codes[3];     // q8, k8, v8 [B][H][N][128]
  float* scales[3];      // [B][H][ceil(N/64)]
  void* y16[3];          // bf16 q, k, v [B][H][N][128] or nullptr
  int B, N, C, H;
};
int launch_qkv_proj_fp8(const QkvProjArgs& a, cudaStream_t s);

// Bounded-wait self-test (wait_selftest.cu).
cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s);

// Builds the tensor maps and launches the BF16 forward kernel.
// Returns 0 on success, a negative dit_status_t otherwise.
int launch_attn_fwd_bf16(const AttnFwdArgs& a, cudaStream_t s);

// Split (compensated) form: q bf16 rotated and split in the kernel, k the
// fp16 split operand [2][B][H][N][D] of launch_prepare_kv_split, v fp16.
struct AttnFwdSplitArgs {
  const void* q;
  const void* k_split;
  const void* v_f16;
  const float* cos;    // [N][64] or nullptr (no rotary embedding)
  const float* sin;
  void* out;
  float* lse;
  int B, H, N;
  bool out_f32;
  int N_kv = 0;     // keys per (b, h); 0: N
};
int launch_attn_fwd_split(const AttnFwdSplitArgs& a, cudaStream_t s);

// cuTensorMapEncodeTiled, resolved once through the runtime's driver entry
// point (no link-time dependency on libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace dit
