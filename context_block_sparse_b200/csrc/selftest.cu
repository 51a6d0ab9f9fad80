// Device self-tests of arithmetic helpers the kernels use (run by the test suite).
#include <cstdint>

#include "sm100.cuh"
#include "splitkv.h"

namespace {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float a, b;
    splitkv::sm100::exp2_poly2(x[i], x[i + 1], a, b);
    y[i] = a;
    y[i + 1] = b;
  } else if (i < n) {
    float a, b;
    splitkv::sm100::exp2_poly2(x[i], x[i], a, b);
    y[i] = a;
  }
}

}  // namespace

extern "C" int splitkv_selftest_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0 || n > (int64_t(1) << 30)) return SPLITKV_ERR_INVALID_ARG;
  if (n == 0) return SPLITKV_OK;
  const int threads = 256;
  const int blocks = int((n / 2 + threads) / threads);
  exp2_poly_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, int(n));
  if (cudaGetLastError() != cudaSuccess) return SPLITKV_ERR_CUDA;
  return SPLITKV_OK;
}
