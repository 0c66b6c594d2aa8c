// Self-test of the bounded waits every kernel of the library uses: one thread
// waits for a barrier phase that nothing completes; after limit_ns the wait
// gives up, records DIT_ERR_TIMEOUT in the device status word and the kernel
// returns, leaving the context usable.
#include "launch.h"
#include "ptx.cuh"

namespace dit {
namespace {

__global__ void wait_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t never;             // initialised for one arrival that never comes
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    abort = 0;
    fence_mbar_init();
    const WaitCtx wc{&abort, status, 0};
    mbar_wait(&never, 0, wc, limit_ns);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s) {
  int* status = device_status_word();
  if (status == nullptr) return cudaErrorInvalidValue;
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace dit
