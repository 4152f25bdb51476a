// numerics.cu -- device-side run of the exponential the softmax kernels use
// (the special-function unit's ex2.approx), so tests can compare it with
// exact values.
#include "lg_common.cuh"
#include "lg_kernels.h"

namespace lg {

__global__ void lg_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, long long n, int method) {
  const long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  (void)method;
  y[k] = ex2_approx(x[k]);
}

cudaError_t launch_exp2(const float* x, float* y, long long n, int method, cudaStream_t stream) {
  const long long blocks = (n + 255) / 256;
  lg_exp2_kernel<<<(unsigned int)blocks, 256, 0, stream>>>(x, y, n, method);
  return cudaGetLastError();
}

// The bounded-wait failure path, end to end: one thread waits on an mbarrier
// that nothing ever arrives on, gives up after `limit` cycles and records
// kErrSelfTest in the device error word; the context stays usable.
__global__ void lg_wait_selftest_kernel(long long limit, unsigned int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_limit(&bar, 0, limit)) atomicOr(err, kErrSelfTest);
  }
}

cudaError_t launch_wait_selftest(long long limit, unsigned int* err, cudaStream_t stream) {
  lg_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit, err);
  return cudaGetLastError();
}

}  // namespace lg
