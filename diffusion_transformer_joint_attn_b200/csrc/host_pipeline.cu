// Attention on q, k, v that live in host memory: the library moves them
// through a caller-provided device workspace in chunks of heads, with the
// host-to-device copies, the kernels and the device-to-host copies of
// consecutive chunks overlapping (three workspace buffers, two copy streams,
// the kernels on the caller's stream).  With pinned host memory the step
// then takes about as long as the larger of its copies, not their sum.
#include <algorithm>
#include <mutex>

#include "launch.h"

namespace dit {
namespace {

constexpr int kMaxDevices = 64;
// Three buffers: while chunk c is copied in, chunk c-1 can be computing and
// chunk c-2 copying out, so the copy-in stream never waits for a buffer when
// compute + copy-out of a chunk take as long as its copy-in.
constexpr int kBuffers = 3;

// Copy streams and the events that order one buffer's chunk: loaded (host to
// device done), computed (kernels done), stored (device to host done).
struct CopyEngines {
  bool ready = false;
  cudaStream_t h2d = nullptr;
  cudaStream_t d2h = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t loaded[kBuffers] = {};
  cudaEvent_t computed[kBuffers] = {};
  cudaEvent_t stored[kBuffers] = {};
  // recorded at the end of each copy stream when an enqueue fails part-way
  cudaEvent_t h2d_tail = nullptr;
  cudaEvent_t d2h_tail = nullptr;
};
CopyEngines g_engines[kMaxDevices];
std::mutex g_mu;   // one enqueue sequence at a time (the events are shared)

cudaError_t engines_for(int dev, CopyEngines** out) {
  CopyEngines& e = g_engines[dev];
  if (!e.ready) {
    cudaError_t r = cudaStreamCreateWithFlags(&e.h2d, cudaStreamNonBlocking);
    if (r == cudaSuccess) r = cudaStreamCreateWithFlags(&e.d2h, cudaStreamNonBlocking);
    if (r == cudaSuccess) r = cudaEventCreateWithFlags(&e.start, cudaEventDisableTiming);
    if (r == cudaSuccess) r = cudaEventCreateWithFlags(&e.h2d_tail, cudaEventDisableTiming);
    if (r == cudaSuccess) r = cudaEventCreateWithFlags(&e.d2h_tail, cudaEventDisableTiming);
    for (int b = 0; b < kBuffers && r == cudaSuccess; ++b) {
      r = cudaEventCreateWithFlags(&e.loaded[b], cudaEventDisableTiming);
      if (r == cudaSuccess) r = cudaEventCreateWithFlags(&e.computed[b], cudaEventDisableTiming);
      if (r == cudaSuccess) r = cudaEventCreateWithFlags(&e.stored[b], cudaEventDisableTiming);
    }
    if (r != cudaSuccess) return r;
    e.ready = true;
  }
  *out = &e;
  return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// A launcher's dit status as a runtime error (the launch's own error if it
// recorded one).
cudaError_t launch_status(int rc) {
  if (rc == 0) return cudaSuccess;
  const cudaError_t e = cudaGetLastError();
  return e != cudaSuccess ? e : cudaErrorInvalidValue;
}

// Offsets of one buffer's arrays for `heads` heads of N tokens.
struct BufferLayout {
  size_t q, k, v, k_rot, v16, out, lse, bytes;
};
BufferLayout buffer_layout(int heads, int N, bool out_f32) {
  const size_t elems = static_cast<size_t>(heads) * N * 128;
  BufferLayout L;
  size_t o = 0;
  L.q = o;
  o += align256(elems * 2);
  L.k = o;
  o += align256(elems * 2);
  L.v = o;
  o += align256(elems * 2);
  L.k_rot = o;
  o += align256(elems * 2);
  L.v16 = o;
  o += align256(elems * 2);
  L.out = o;
  o += align256(elems * (out_f32 ? 4 : 2));
  L.lse = o;
  o += align256(static_cast<size_t>(heads) * N * 4);
  L.bytes = o;
  return L;
}

// Workspace of dit_attn_forward_host_static: one array in the library's
// device image, shared by every call on a device.  Every byte of it is
// written (by a copy or a kernel) before it is read, so nothing needs
// clearing.
__device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

}  // namespace

cudaError_t static_workspace(void** out) {
  static void* cached[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t r = cudaGetDevice(&dev);
  if (r != cudaSuccess) return r;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == nullptr) {
    // with device `dev` current: the array's address in this device's copy of the image
    void* ptr = nullptr;
    if ((r = cudaGetSymbolAddress(&ptr, g_static_workspace)) != cudaSuccess) return r;
    cached[dev] = ptr;
  }
  *out = cached[dev];
  return cudaSuccess;
}

size_t host_forward_workspace_bytes(int BH, int N, int chunk_heads, bool out_f32) {
  const int heads = std::min(chunk_heads, BH);
  return kBuffers * buffer_layout(heads, N, out_f32).bytes;
}

namespace {

// The enqueue sequence of host_forward; on failure it returns at once, leaving
// whatever it queued on the copy streams.
cudaError_t host_forward_enqueue(const HostForwardArgs& a, cudaStream_t s, CopyEngines* e);

}  // namespace

cudaError_t host_forward(const HostForwardArgs& a, cudaStream_t s) {
  int dev = 0;
  cudaError_t r = cudaGetDevice(&dev);
  if (r != cudaSuccess) return r;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  CopyEngines* e = nullptr;
  if ((r = engines_for(dev, &e)) != cudaSuccess) return r;
  r = host_forward_enqueue(a, s, e);
  if (r != cudaSuccess) {
    // An enqueue failed part-way: copies already queued on the private copy
    // streams still read the caller's host buffers and write its results.
    // Order them before `stream` (best effort; the first error is the one
    // returned), so that a caller who synchronises `stream` after the error
    // may free or reuse those buffers.
    if (cudaEventRecord(e->h2d_tail, e->h2d) == cudaSuccess) cudaStreamWaitEvent(s, e->h2d_tail, 0);
    if (cudaEventRecord(e->d2h_tail, e->d2h) == cudaSuccess) cudaStreamWaitEvent(s, e->d2h_tail, 0);
  }
  return r;
}

namespace {

cudaError_t host_forward_enqueue(const HostForwardArgs& a, cudaStream_t s, CopyEngines* e) {
  cudaError_t r = cudaSuccess;
  const int BH = a.B * a.H;
  const int chunk = std::min(a.chunk_heads, BH);
  const BufferLayout L = buffer_layout(chunk, a.N, a.out_f32);
  const size_t head_elems = static_cast<size_t>(a.N) * 128;
  const size_t out_esize = a.out_f32 ? 4 : 2;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);

  // work the caller queued before this call (e.g. the rotary tables, or an
  // earlier use of the workspace) precedes every copy of this call
  if ((r = cudaEventRecord(e->start, s)) != cudaSuccess) return r;
  if ((r = cudaStreamWaitEvent(e->h2d, e->start, 0)) != cudaSuccess) return r;

  // chunks: one head first and one head last (the copy-in before the first
  // kernel and the kernel + copy-out after the last copy-in are not hidden;
  // small end chunks keep them short), `chunk` heads in between
  const bool ramp = BH > 2 && chunk > 1;
  int c = 0;
  for (int h0 = 0; h0 < BH; ++c) {
    int hc;
    if (!ramp)
      hc = std::min(chunk, BH - h0);
    else if (h0 == 0 || h0 == BH - 1)
      hc = 1;
    else
      hc = std::min(chunk, BH - 1 - h0);   // the last head is kept for the final chunk
    const int b = c % kBuffers;
    uint8_t* base = ws + static_cast<size_t>(b) * L.bytes;
    const size_t in_off = static_cast<size_t>(h0) * head_elems * 2;
    const size_t in_bytes = static_cast<size_t>(hc) * head_elems * 2;
    // the buffer's previous chunk (of this call or of the previous one) has left the device
    if ((r = cudaStreamWaitEvent(e->h2d, e->stored[b], 0)) != cudaSuccess) return r;
    const void* src[3] = {a.q, a.k, a.v};
    const size_t dst[3] = {L.q, L.k, L.v};
    for (int i = 0; i < 3; ++i) {
      r = cudaMemcpyAsync(base + dst[i], static_cast<const uint8_t*>(src[i]) + in_off, in_bytes,
                          cudaMemcpyHostToDevice, e->h2d);
      if (r != cudaSuccess) return r;
    }
    if ((r = cudaEventRecord(e->loaded[b], e->h2d)) != cudaSuccess) return r;
    if ((r = cudaStreamWaitEvent(s, e->loaded[b], 0)) != cudaSuccess) return r;

    float* lse = a.lse != nullptr ? reinterpret_cast<float*>(base + L.lse) : nullptr;
    if (a.cos != nullptr) {
      PrepareKVArgs p{base + L.k, base + L.v, a.cos, a.sin, base + L.k_rot, base + L.v16, 1, hc, a.N, 128};
      if ((r = launch_prepare_kv(p, s)) != cudaSuccess) return r;
      AttnFwdArgs f{base + L.q, base + L.k_rot, base + L.v16, a.cos, a.sin, base + L.out, lse, 1, hc, a.N,
                    a.out_f32, true, true};
      if ((r = launch_status(launch_attn_fwd_bf16(f, s))) != cudaSuccess) return r;
    } else {
      AttnFwdArgs f{base + L.q, base + L.k, base + L.v, nullptr, nullptr, base + L.out, lse, 1, hc, a.N,
                    a.out_f32, false, false};
      if ((r = launch_status(launch_attn_fwd_bf16(f, s))) != cudaSuccess) return r;
    }
    if ((r = cudaEventRecord(e->computed[b], s)) != cudaSuccess) return r;
    if ((r = cudaStreamWaitEvent(e->d2h, e->computed[b], 0)) != cudaSuccess) return r;
    r = cudaMemcpyAsync(static_cast<uint8_t*>(a.out) + static_cast<size_t>(h0) * head_elems * out_esize,
                        base + L.out, static_cast<size_t>(hc) * head_elems * out_esize, cudaMemcpyDeviceToHost,
                        e->d2h);
    if (r != cudaSuccess) return r;
    if (a.lse != nullptr) {
      r = cudaMemcpyAsync(a.lse + static_cast<size_t>(h0) * a.N, lse, static_cast<size_t>(hc) * a.N * 4,
                          cudaMemcpyDeviceToHost, e->d2h);
      if (r != cudaSuccess) return r;
    }
    if ((r = cudaEventRecord(e->stored[b], e->d2h)) != cudaSuccess) return r;
    h0 += hc;
  }
  // the caller's stream completes only after the results are on the host
  for (int b = 0; b < kBuffers; ++b)
    if ((r = cudaStreamWaitEvent(s, e->stored[b], 0)) != cudaSuccess) return r;
  return cudaSuccess;
}

}  // namespace

}  // namespace dit
