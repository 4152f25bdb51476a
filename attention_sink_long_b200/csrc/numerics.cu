// numerics.cu -- device-side run of the exponential the softmax kernels use,
// so tests can compare it with exact values and with the hardware ex2.approx.
#include "lg_common.cuh"
#include "lg_kernels.h"

namespace lg {

__global__ void lg_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, long long n, int method) {
  const long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  if (method == 2) {
    // the paired form the forward softmax runs (two lanes of work per instruction)
    const long long k2 = ((k ^ 1LL) < n) ? (k ^ 1LL) : k;
    const float2 r = ex2_poly2(make_float2(x[k], x[k2]));
    y[k] = r.x;
  } else {
    y[k] = method == 1 ? ex2_poly(x[k]) : ex2_approx(x[k]);
  }
}

cudaError_t launch_exp2(const float* x, float* y, long long n, int method, cudaStream_t stream) {
  const long long blocks = (n + 255) / 256;
  lg_exp2_kernel<<<(unsigned int)blocks, 256, 0, stream>>>(x, y, n, method);
  return cudaGetLastError();
}

}  // namespace lg
