// Self-test of the kernels' failure detection. One launch waits on an
// mbarrier that nothing arrives at, with the same bounded wait as the GEMV
// kernels' stage rings but a caller-given time limit; the wait gives up,
// records a timeout in the device error word and the kernel returns, so the
// host reads TERN_ETIMEOUT from tern_device_error() and the context stays
// usable. Nothing faults, traps or hangs: the wait always ends.
#include <cuda_runtime.h>

#include "tern_internal.h"
#include "tern_ptx.cuh"

namespace tern {

int read_clear_dev_error_selftest(void* stream, unsigned* out) { return read_clear_dev_error_tu(stream, out); }

namespace {

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // phase 0 of `bar` never completes (its one expected arrival never comes)
  if (threadIdx.x == 0) (void)mbar_wait_bounded_ns(&bar, 0u, limit_ns);
  __syncthreads();
}

}  // namespace
}  // namespace tern

extern "C" tern_status tern_selftest_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > tern::kWaitLimitNs) return TERN_EINVAL;
  tern::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ECUDA;
}
