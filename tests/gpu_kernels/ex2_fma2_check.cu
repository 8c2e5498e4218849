// Test kernel (built by tests/test_gpu_ex2.py, not part of the library): the
// attention softmax's FMA-pipe exponential next to CUDA's exp2f, element by
// element, so the two can be compared on the device that runs them.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ex2_fma.cuh"

__global__ void ex2_pair_kernel(const float* __restrict__ x, float* __restrict__ y_fma, float* __restrict__ y_hw,
                                int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);  // first element of this thread's pair
  if (i + 1 < n) {
    float p0, p1;
    sda::ex2_fma2(x[i], x[i + 1], p0, p1);
    y_fma[i] = p0;
    y_fma[i + 1] = p1;
    y_hw[i] = exp2f(x[i]);
    y_hw[i + 1] = exp2f(x[i + 1]);
  }
}

// x, y_fma, y_hw: n floats of device memory, n even. 0 on success.
extern "C" int ex2_check(const float* x, float* y_fma, float* y_hw, int n) {
  if (n <= 0 || (n & 1) != 0 || x == nullptr || y_fma == nullptr || y_hw == nullptr) return -1;
  const int pairs = n / 2;
  ex2_pair_kernel<<<(pairs + 255) / 256, 256>>>(x, y_fma, y_hw, n);
  if (cudaGetLastError() != cudaSuccess) return -2;
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : -3;
}
