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
// y[i] = exp2_fma_pipe(x[i]): the FMA-pipe exponential the softmax kernels use for part of
// their exponentials, evaluated element by element for a check against 2^x.
__global__ void __launch_bounds__(256) fa_selftest_exp2_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float a = x[i], b = x[i];
  exp2_fma_pipe(a, b);
  y[i] = a;
}
}  // namespace

cudaError_t launch_selftest_exp2(const float* x, float* y, int n, cudaStream_t s) {
  fa_selftest_exp2_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int* err, cudaStream_t s) {
  fa_selftest_wait_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}
}  // namespace fa
