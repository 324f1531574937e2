// Failure-detection self-test: one thread waits, with the library's bounded wait, on an
// mbarrier that nothing signals. The wait runs out after the given limit, records the timeout
// in the device status word (as a stalled pipeline would) and returns; the kernel then exits
// normally, so the context stays usable. No fault, trap or unbounded wait is involved.
#include "osc_device.cuh"
#include "osc_internal.h"

namespace osc {

__global__ void selftest_wait_kernel(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    mbar_wait(smem_u32(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), status, limit_ns);
  }
}

cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace osc
