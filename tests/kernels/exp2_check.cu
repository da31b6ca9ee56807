// Test harness: evaluates the attention kernel's FMA-pipe exp2 and CUDA's
// exp2f on the same inputs (built and loaded by tests/test_gpu_exp2.py).
#include <cuda_runtime.h>

#include "exp2_fma.cuh"

__global__ void eval_kernel(const float* x, float* approx, float* ref, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i + 1 < n) {
    const float2 r = rkv::exp2_fma2(make_float2(x[2 * i], x[2 * i + 1]));
    approx[2 * i] = r.x;
    approx[2 * i + 1] = r.y;
    ref[2 * i] = exp2f(x[2 * i]);
    ref[2 * i + 1] = exp2f(x[2 * i + 1]);
  }
}

extern "C" int exp2_check(const float* x_dev, float* approx_dev, float* ref_dev, int n) {
  eval_kernel<<<(n / 2 + 255) / 256, 256>>>(x_dev, approx_dev, ref_dev, n);
  return int(cudaDeviceSynchronize());
}
