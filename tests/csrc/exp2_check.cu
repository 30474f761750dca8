// Test-only kernel: evaluates the prefill softmax's FMA-pipe exp2 and the
// SFU exp2 on device next to CUDA's exp2f, for tests/test_gpu_exp2.py.
#include <cuda_runtime.h>

#include "swa_common.cuh"
#include "swa_exp2.cuh"

__global__ void exp2_check_kernel(const float* x, float* fma_pipe, float* sfu, float* ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n) return;
  float a = x[i], b = x[i + 1];
  swa::exp2_fma_pipe(a, b);
  fma_pipe[i] = a;
  fma_pipe[i + 1] = b;
  sfu[i] = swa::fast_exp2(x[i]);
  sfu[i + 1] = swa::fast_exp2(x[i + 1]);
  ref[i] = exp2f(x[i]);
  ref[i + 1] = exp2f(x[i + 1]);
}

extern "C" int exp2_check(const float* x, float* fma_pipe, float* sfu, float* ref, int n) {
  exp2_check_kernel<<<(n / 2 + 255) / 256, 256>>>(x, fma_pipe, sfu, ref, n);
  if (cudaGetLastError() != cudaSuccess) return 1;
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}
