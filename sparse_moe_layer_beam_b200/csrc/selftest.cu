// selftest.cu - a device-side check of the failure path every tensor-core
// kernel of this library takes when a bounded wait runs out: one thread waits
// on an mbarrier that nothing completes, gives up after the limit, records a
// status bit in the workspace and returns. The context stays usable.
#include "internal.h"
#include "sm100.cuh"

namespace beam {
namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(unsigned* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  // phase 0 of a fresh barrier never completes: nothing arrives on it
  if (threadIdx.x == 0)
    mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status, kFlagSelftest,
              limit_ns);
  __syncwarp();
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned* status, int limit_ms, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(status, (uint64_t)limit_ms * 1000000ull);
  return cudaGetLastError();
}

}  // namespace beam
