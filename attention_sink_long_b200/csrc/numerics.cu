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

}  // namespace lg
