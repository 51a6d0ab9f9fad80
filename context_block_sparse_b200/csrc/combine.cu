// The exchange step of Split-KV over several ranks (news page, "Exchange the
// smaller side"): every rank holds a share of the context's keys and computes
// every query row's exact partial result over them; the owner of a query row
// receives the ranks' results for it, and these kernels combine them.
//
//   combine: per query row and head, from R results (O_r, LSE_r) -- O_r the
//     softmax-weighted mean over rank r's keys, LSE_r their log-sum-exp --
//     M = max_r LSE_r, w_r = exp(LSE_r - M), O = sum_r w_r O_r / sum_r w_r,
//     LSE = M + log(sum_r w_r); a row with every LSE_r = -inf gets O = 0,
//     LSE = -inf.
//   sum: out = sum_r part_r, ranks in ascending order (the dQ shares).
//
// Both are streaming, HBM-bound passes: one thread per 4 consecutive floats of a
// row (16-byte loads, consecutive threads on consecutive addresses), a grid of a
// few waves over the SMs, ranks summed in a fixed order (run-to-run identical).
#include <cmath>
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
    combine_kernel(int R, int64_t rows, int d4, const float4* __restrict__ o_parts,
                   const float* __restrict__ lse_parts, void* __restrict__ o, int o_bf16,
                   float* __restrict__ lse) {
  const int64_t units = rows * d4;
  for (int64_t u = int64_t(blockIdx.x) * kThreads + threadIdx.x; u < units; u += int64_t(gridDim.x) * kThreads) {
    const int64_t row = u / d4;
    const int c = int(u - row * d4);
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, __ldg(lse_parts + int64_t(r) * rows + row));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    if (M != -INFINITY) {
      for (int r = 0; r < R; ++r) {
        const float lr = __ldg(lse_parts + int64_t(r) * rows + row);
        if (lr == -INFINITY) continue;   // rank r holds no key of this row
        const float w = expf(lr - M);
        const float4 x = __ldg(o_parts + (int64_t(r) * rows + row) * d4 + c);
        acc.x = fmaf(w, x.x, acc.x);
        acc.y = fmaf(w, x.y, acc.y);
        acc.z = fmaf(w, x.z, acc.z);
        acc.w = fmaf(w, x.w, acc.w);
        L += w;
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if (o_bf16) {
      uint2 p;
      p.x = splitkv::pack_bf16(acc.x * inv, acc.y * inv);
      p.y = splitkv::pack_bf16(acc.z * inv, acc.w * inv);
      reinterpret_cast<uint2*>(o)[row * d4 + c] = p;
    } else {
      reinterpret_cast<float4*>(o)[row * d4 + c] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (c == 0) lse[row] = L > 0.f ? M + logf(L) : -INFINITY;
  }
}

__global__ void __launch_bounds__(kThreads)
    sum_kernel(int R, int64_t n4, const float4* __restrict__ parts, float4* __restrict__ out) {
  for (int64_t u = int64_t(blockIdx.x) * kThreads + threadIdx.x; u < n4; u += int64_t(gridDim.x) * kThreads) {
    float4 acc = __ldg(parts + u);
    for (int r = 1; r < R; ++r) {
      const float4 x = __ldg(parts + int64_t(r) * n4 + u);
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    out[u] = acc;
  }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int splitkv_combine_ranks(int32_t num_ranks, int64_t rows, int32_t head_dim, const float* o_parts,
                                     const float* lse_parts, void* o, int o_dtype, float* lse, void* stream) {
  if (num_ranks < 1 || num_ranks > SPLITKV_MAX_RANKS || rows < 0 || head_dim < 4 || head_dim % 4 ||
      (o_dtype != SPLITKV_DTYPE_F32 && o_dtype != SPLITKV_DTYPE_BF16))
    return SPLITKV_ERR_INVALID_ARG;
  if (rows == 0) return SPLITKV_OK;
  if (!o_parts || !lse_parts || !o || !lse || !aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(lse, 4) ||
      !aligned(o, o_dtype == SPLITKV_DTYPE_F32 ? 16 : 8))
    return SPLITKV_ERR_INVALID_ARG;
  const int d4 = head_dim / 4;
  if (rows > (int64_t(1) << 40) / d4) return SPLITKV_ERR_INVALID_ARG;
  combine_kernel<<<grid_for(rows * d4), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      num_ranks, rows, d4, reinterpret_cast<const float4*>(o_parts), lse_parts, o, o_dtype == SPLITKV_DTYPE_BF16,
      lse);
  return cudaGetLastError() == cudaSuccess ? SPLITKV_OK : SPLITKV_ERR_CUDA;
}

extern "C" int splitkv_enable_peer_access(int32_t peer_device) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPLITKV_ERR_CUDA;
  if (peer_device == dev) return SPLITKV_OK;
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess) return SPLITKV_ERR_CUDA;
  if (peer_device < 0 || peer_device >= n) return SPLITKV_ERR_INVALID_ARG;
  int can = 0;
  if (cudaDeviceCanAccessPeer(&can, dev, peer_device) != cudaSuccess) return SPLITKV_ERR_CUDA;
  if (!can) return SPLITKV_ERR_UNSUPPORTED;
  const cudaError_t e = cudaDeviceEnablePeerAccess(peer_device, 0);
  if (e == cudaErrorPeerAccessAlreadyEnabled) {
    cudaGetLastError();   // clear the (non-sticky) error the call left: access is on, as asked
    return SPLITKV_OK;
  }
  return e == cudaSuccess ? SPLITKV_OK : SPLITKV_ERR_CUDA;
}

extern "C" int splitkv_sum_ranks(int32_t num_ranks, int64_t n, const float* parts, float* out, void* stream) {
  if (num_ranks < 1 || num_ranks > SPLITKV_MAX_RANKS || n < 0 || n % 4 || n > (int64_t(1) << 42))
    return SPLITKV_ERR_INVALID_ARG;
  if (n == 0) return SPLITKV_OK;
  if (!parts || !out || !aligned(parts, 16) || !aligned(out, 16)) return SPLITKV_ERR_INVALID_ARG;
  sum_kernel<<<grid_for(n / 4), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      num_ranks, n / 4, reinterpret_cast<const float4*>(parts), reinterpret_cast<float4*>(out));
  return cudaGetLastError() == cudaSuccess ? SPLITKV_OK : SPLITKV_ERR_CUDA;
}
