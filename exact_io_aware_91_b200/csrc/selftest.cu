// Self-test of the bounded waits every kernel of the library uses: one CTA, one thread
// waits on an mbarrier that nothing ever arrives at, through the same helper (mbar_wait).
// The wait must give up after its wall-time limit, record the timeout in the device error
// word (read back by fa_device_status) and return, leaving the context usable -- the
// failure path of the real kernels, exercised without any fault, trap or hang.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {
__global__ void __launch_bounds__(32) fa_selftest_wait_kernel(int* err) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(bar, 1);  // expects one arrival that never comes
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const WaitCtx w{reinterpret_cast<volatile int*>(&abort_flag), err};
    (void)mbar_wait(bar, 0, w);  // bounded: returns false and sets the error word
  }
}
}  // namespace

cudaError_t launch_selftest_wait(int* err, cudaStream_t s) {
  fa_selftest_wait_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}
}  // namespace fa
