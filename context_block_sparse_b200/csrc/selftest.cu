// Device self-tests of helpers the kernels use (run by the test suite): the FMA-pipe
// exp2, and the bounded mbarrier wait that turns a wait nothing completes into a
// recorded SPLITKV_ERR_TIMEOUT instead of a hang.
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

// An mbarrier no one ever arrives on: thread 0 and all of warp 1 wait for its first phase
// with the kernels' bounded waits.  Thread 0 gives up after the time limit and records
// SPLITKV_ERR_TIMEOUT with its site in status[0..1]; warp 1 stops on the abort flag that
// sets (or on its own limit).
__global__ void wait_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    splitkv::sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    splitkv::sm100::mbar_fence_init();
  }
  __syncthreads();
  const splitkv::sm100::WaitCtx c{&abort_flag, status, splitkv::sm100::kWaitLimitNs};
  if (threadIdx.x == 0)
    splitkv::sm100::mbar_wait(&bar, 0, c, 9 * 10000 + __LINE__);
  else if (threadIdx.x >= 32)
    splitkv::sm100::warp_wait(&bar, 0, c, 9 * 10000 + __LINE__);
  __syncthreads();
}

}  // namespace

extern "C" int splitkv_selftest_wait_timeout(int32_t* status_out, void* stream) {
  if (!status_out) return SPLITKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* d = nullptr;
  if (cudaMalloc(&d, 2 * sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return SPLITKV_ERR_NO_MEMORY;
  }
  int h[2] = {0, 0};
  int st = SPLITKV_OK;
  if (cudaMemsetAsync(d, 0, sizeof(h), s) != cudaSuccess) st = SPLITKV_ERR_CUDA;
  if (st == SPLITKV_OK) {
    wait_timeout_kernel<<<1, 64, 0, s>>>(d);
    if (cudaGetLastError() != cudaSuccess) st = SPLITKV_ERR_CUDA;
  }
  if (st == SPLITKV_OK && cudaMemcpyAsync(h, d, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    st = SPLITKV_ERR_CUDA;
  if (st == SPLITKV_OK && cudaStreamSynchronize(s) != cudaSuccess) st = SPLITKV_ERR_CUDA;
  cudaFree(d);
  status_out[0] = h[0];
  status_out[1] = h[1];
  return st;
}

extern "C" int splitkv_selftest_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0 || n > (int64_t(1) << 30)) return SPLITKV_ERR_INVALID_ARG;
  if (n == 0) return SPLITKV_OK;
  const int threads = 256;
  const int blocks = int((n / 2 + threads) / threads);
  exp2_poly_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, int(n));
  if (cudaGetLastError() != cudaSuccess) return SPLITKV_ERR_CUDA;
  return SPLITKV_OK;
}
