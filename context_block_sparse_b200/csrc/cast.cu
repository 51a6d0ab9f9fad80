// Output conversion: float32 result arrays (o, dq, dk, dv, dkb, dvb) to bfloat16 for
// callers that keep activations and gradients in bf16.  Not a step of the method: the
// kernels compute and accumulate in fp32; this rounds the finished arrays (round to
// nearest even, the conversion cuda_bf16.h provides) so that half the bytes leave the
// GPU.  A streaming, HBM-bound pass: 8 elements per thread step (two 16-byte loads,
// one 16-byte store), a grid of a few waves over the SMs.
#include <cstdint>

#include "common.cuh"
#include "splitkv.h"

namespace {

constexpr int kThreads = 256;

int grid_for(int64_t units) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (units + kThreads - 1) / kThreads;
  const int64_t cap = int64_t(sms) * 8;
  return int(want < cap ? (want > 0 ? want : 1) : cap);
}

__global__ void __launch_bounds__(kThreads)
    cast_bf16_x8_kernel(int64_t n8, const float4* __restrict__ src, uint4* __restrict__ dst) {
  for (int64_t u = int64_t(blockIdx.x) * kThreads + threadIdx.x; u < n8; u += int64_t(gridDim.x) * kThreads) {
    const float4 a = __ldg(src + 2 * u), b = __ldg(src + 2 * u + 1);
    dst[u] = make_uint4(splitkv::pack_bf16(a.x, a.y), splitkv::pack_bf16(a.z, a.w), splitkv::pack_bf16(b.x, b.y),
                        splitkv::pack_bf16(b.z, b.w));
  }
}

__global__ void __launch_bounds__(kThreads)
    cast_bf16_kernel(int64_t i0, int64_t n, const float* __restrict__ src, uint16_t* __restrict__ dst) {
  for (int64_t i = i0 + int64_t(blockIdx.x) * kThreads + threadIdx.x; i < n; i += int64_t(gridDim.x) * kThreads) {
    const __nv_bfloat16 h = __float2bfloat16_rn(src[i]);
    dst[i] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int splitkv_cast_bf16(int64_t n, const float* src, uint16_t* dst, void* stream) {
  if (n < 0 || n > (int64_t(1) << 42)) return SPLITKV_ERR_INVALID_ARG;
  if (n == 0) return SPLITKV_OK;
  if (!src || !dst) return SPLITKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int64_t i0 = 0;
  if (aligned16(src) && aligned16(dst) && n >= 8) {
    const int64_t n8 = n / 8;
    cast_bf16_x8_kernel<<<grid_for(n8), kThreads, 0, s>>>(n8, reinterpret_cast<const float4*>(src),
                                                          reinterpret_cast<uint4*>(dst));
    if (cudaGetLastError() != cudaSuccess) return SPLITKV_ERR_CUDA;
    i0 = n8 * 8;
  }
  if (i0 < n) {
    cast_bf16_kernel<<<grid_for(n - i0), kThreads, 0, s>>>(i0, n, src, dst);
    if (cudaGetLastError() != cudaSuccess) return SPLITKV_ERR_CUDA;
  }
  return SPLITKV_OK;
}
