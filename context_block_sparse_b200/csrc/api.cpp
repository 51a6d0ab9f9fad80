// C-ABI attention entry points of libsplitkv.so: argument checks, workspace
// carving and kernel dispatch.  Every step of the computation runs in the
// sm_100a kernels; this file only validates and launches.
#include <cstdint>
#include <new>

#include "splitkv.h"
#include "splitkv_internal.h"

namespace {

using splitkv::all_aligned16;
using splitkv::block_ptrs_ok;
using splitkv::check_plan;
using splitkv::DevPlan;
using splitkv::rec_bytes;

bool aligned(const void* p, uintptr_t a) { return splitkv::ptr_aligned(p, a); }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPLITKV_OK;
  cudaGetLastError();
  return SPLITKV_ERR_CUDA;
}

}  // namespace

extern "C" {

int splitkv_attn_fwd(const splitkv_plan_t* plan, const void* q, const void* k, const void* v, float scale,
                     void* ws, size_t ws_bytes, void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  if (!all_aligned16(q, k, v, ws)) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::FwdWs L = splitkv::fwd_ws_layout(dp->E, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  char* w = static_cast<char*>(ws);
  return cuda_status(splitkv::launch_fwd_partial(
      *dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
      scale, static_cast<void*>(w + L.o_off), reinterpret_cast<float*>(w + L.m_off),
      reinterpret_cast<float*>(w + L.l_off), static_cast<cudaStream_t>(stream)));
}

int splitkv_merge(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb, float scale,
                  const void* ws, size_t ws_bytes, void* o, int o_dtype, float* lse, void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  if (!all_aligned16(q, ws, o) || !block_ptrs_ok(dp, kb, vb) || !lse || !aligned(lse, 4))
    return SPLITKV_ERR_INVALID_ARG;
  if (o_dtype != SPLITKV_DTYPE_F32 && o_dtype != SPLITKV_DTYPE_BF16) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::FwdWs L = splitkv::fwd_ws_layout(dp->E, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  const char* w = static_cast<const char*>(ws);
  return cuda_status(splitkv::launch_merge(
      *dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kb), static_cast<const uint16_t*>(vb),
      scale, static_cast<const void*>(w + L.o_off), reinterpret_cast<const float*>(w + L.m_off),
      reinterpret_cast<const float*>(w + L.l_off), o, o_dtype == SPLITKV_DTYPE_BF16 ? 1 : 0, lse,
      static_cast<cudaStream_t>(stream)));
}

int splitkv_merge_to_owners(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb, float scale,
                            const void* ws, size_t ws_bytes, int32_t num_ranks, int32_t rank,
                            float* const* o_dest, float* const* lse_dest, void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  int R = 1, self = 0;
  splitkv::plan_ranks(plan, &R, &self);
  if (num_ranks != R || rank != self || !o_dest || !lse_dest || !aligned(o_dest, 8) || !aligned(lse_dest, 8))
    return SPLITKV_ERR_INVALID_ARG;
  if (!all_aligned16(q, ws) || !block_ptrs_ok(dp, kb, vb)) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::FwdWs L = splitkv::fwd_ws_layout(dp->E, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  const char* w = static_cast<const char*>(ws);
  return cuda_status(splitkv::launch_merge(
      *dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kb), static_cast<const uint16_t*>(vb),
      scale, static_cast<const void*>(w + L.o_off), reinterpret_cast<const float*>(w + L.m_off),
      reinterpret_cast<const float*>(w + L.l_off), nullptr, 0, nullptr, static_cast<cudaStream_t>(stream),
      splitkv::MergeDest{o_dest, lse_dest, R, self}));
}

int splitkv_bwd_delta(const splitkv_plan_t* plan, const void* o, int o_dtype, const void* dout, void* ws,
                      size_t ws_bytes, void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  if (!all_aligned16(o, dout, ws)) return SPLITKV_ERR_INVALID_ARG;
  if (o_dtype != SPLITKV_DTYPE_F32 && o_dtype != SPLITKV_DTYPE_BF16) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::BwdWs L = splitkv::bwd_ws_layout(dp->E, dp->Nq, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  float* delta = reinterpret_cast<float*>(static_cast<char*>(ws) + L.delta_off);
  return cuda_status(splitkv::launch_bwd_delta(*dp, o, o_dtype == SPLITKV_DTYPE_BF16 ? 1 : 0,
                                               static_cast<const uint16_t*>(dout), delta,
                                               static_cast<cudaStream_t>(stream)));
}

namespace {
int bwd_partial_part(const splitkv_plan_t* plan, const void* q, const void* k, const void* v, const float* lse,
                     const void* dout, float* dk, float* dv, float scale, void* ws, size_t ws_bytes, void* stream,
                     int which) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  if (!all_aligned16(q, k, v, dout, ws) || !lse || !aligned(lse, 4)) return SPLITKV_ERR_INVALID_ARG;
  if (which != 2 && !all_aligned16(dk, dv)) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::BwdWs L = splitkv::bwd_ws_layout(dp->E, dp->Nq, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  char* w = static_cast<char*>(ws);
  return cuda_status(splitkv::launch_bwd_partial(
      *dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
      static_cast<const uint16_t*>(dout), lse, reinterpret_cast<const float*>(w + L.delta_off), scale, dk, dv,
      reinterpret_cast<float*>(w + L.dq_off), static_cast<cudaStream_t>(stream), which));
}
}  // namespace

int splitkv_bwd_partial(const splitkv_plan_t* plan, const void* q, const void* k, const void* v, const float* lse,
                        const void* dout, float* dk, float* dv, float scale, void* ws, size_t ws_bytes,
                        void* stream) {
  return bwd_partial_part(plan, q, k, v, lse, dout, dk, dv, scale, ws, ws_bytes, stream, 0);
}

int splitkv_bwd_dkdv(const splitkv_plan_t* plan, const void* q, const void* k, const void* v, const float* lse,
                     const void* dout, float* dk, float* dv, float scale, void* ws, size_t ws_bytes,
                     void* stream) {
  return bwd_partial_part(plan, q, k, v, lse, dout, dk, dv, scale, ws, ws_bytes, stream, 1);
}

int splitkv_bwd_dq(const splitkv_plan_t* plan, const void* q, const void* k, const void* v, const float* lse,
                   const void* dout, float scale, void* ws, size_t ws_bytes, void* stream) {
  return bwd_partial_part(plan, q, k, v, lse, dout, nullptr, nullptr, scale, ws, ws_bytes, stream, 2);
}

int splitkv_bwd_reduce(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb, const float* lse,
                       const void* dout, float* dq, float* dkb, float* dvb, float scale, const void* ws,
                       size_t ws_bytes, void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  if (!all_aligned16(q, dout, dq, ws) || !block_ptrs_ok(dp, kb, vb, dkb, dvb) || !lse || !aligned(lse, 4))
    return SPLITKV_ERR_INVALID_ARG;
  const splitkv::BwdWs L = splitkv::bwd_ws_layout(dp->E, dp->Nq, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  const char* w = static_cast<const char*>(ws);
  return cuda_status(splitkv::launch_bwd_reduce(
      *dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kb), static_cast<const uint16_t*>(vb),
      static_cast<const uint16_t*>(dout), lse, reinterpret_cast<const float*>(w + L.delta_off),
      static_cast<const void*>(w + L.dq_off), scale, dq, dkb, dvb, static_cast<cudaStream_t>(stream)));
}

int splitkv_bwd_reduce_to_owners(const splitkv_plan_t* plan, const void* q, const void* kb, const void* vb,
                                 const float* lse, const void* dout, float* dkb, float* dvb, float scale,
                                 const void* ws, size_t ws_bytes, int32_t num_ranks, int32_t rank,
                                 float* const* dq_dest, void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  int R = 1, self = 0;
  splitkv::plan_ranks(plan, &R, &self);
  if (num_ranks != R || rank != self || !dq_dest || !aligned(dq_dest, 8)) return SPLITKV_ERR_INVALID_ARG;
  if (!all_aligned16(q, dout, ws) || !block_ptrs_ok(dp, kb, vb, dkb, dvb) || !lse || !aligned(lse, 4))
    return SPLITKV_ERR_INVALID_ARG;
  const splitkv::BwdWs L = splitkv::bwd_ws_layout(dp->E, dp->Nq, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  const char* w = static_cast<const char*>(ws);
  return cuda_status(splitkv::launch_bwd_reduce(
      *dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kb), static_cast<const uint16_t*>(vb),
      static_cast<const uint16_t*>(dout), lse, reinterpret_cast<const float*>(w + L.delta_off),
      static_cast<const void*>(w + L.dq_off), scale, nullptr, dkb, dvb, static_cast<cudaStream_t>(stream),
      splitkv::MergeDest{dq_dest, nullptr, R, self}));
}

int splitkv_attn_bwd(const splitkv_plan_t* plan, const void* q, const void* k, const void* v, const void* kb,
                     const void* vb, const void* o, int o_dtype, const float* lse, const void* dout, float* dq,
                     float* dk, float* dv, float* dkb, float* dvb, float scale, void* ws, size_t ws_bytes,
                     void* stream) {
  const DevPlan* dp = nullptr;
  int st = check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  // check everything up front so that no launch happens on a call that fails
  if (!all_aligned16(q, k, v, o, dout, dq, dk, dv, ws) || !block_ptrs_ok(dp, kb, vb, dkb, dvb) || !lse ||
      !aligned(lse, 4))
    return SPLITKV_ERR_INVALID_ARG;
  if (o_dtype != SPLITKV_DTYPE_F32 && o_dtype != SPLITKV_DTYPE_BF16) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::BwdWs L = splitkv::bwd_ws_layout(dp->E, dp->Nq, dp->bs, dp->Hq, dp->d, rec_bytes(dp));
  if (ws_bytes < L.total) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  st = splitkv_bwd_delta(plan, o, o_dtype, dout, ws, ws_bytes, stream);
  if (st != SPLITKV_OK) return st;
  st = splitkv_bwd_partial(plan, q, k, v, lse, dout, dk, dv, scale, ws, ws_bytes, stream);
  if (st != SPLITKV_OK) return st;
  return splitkv_bwd_reduce(plan, q, kb, vb, lse, dout, dq, dkb, dvb, scale, ws, ws_bytes, stream);
}

int splitkv_plan_status(const splitkv_plan_t* plan, void* stream, int32_t* site) {
  if (!plan) return SPLITKV_ERR_INVALID_ARG;
  const DevPlan* dp = splitkv::plan_device_view(plan);
  if (!dp) return SPLITKV_ERR_NOT_UPLOADED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int words[2] = {0, 0};
  int st = cuda_status(cudaMemcpyAsync(words, dp->status, sizeof(words), cudaMemcpyDeviceToHost, s));
  if (st == SPLITKV_OK) st = cuda_status(cudaStreamSynchronize(s));
  if (st != SPLITKV_OK) return st;
  if (site) *site = words[1];
  if (words[0] == 0 && words[1] == 0) return SPLITKV_OK;
  st = cuda_status(cudaMemsetAsync(dp->status, 0, sizeof(words), s));
  if (st == SPLITKV_OK) st = cuda_status(cudaStreamSynchronize(s));
  return st != SPLITKV_OK ? st : (words[0] != 0 ? words[0] : SPLITKV_ERR_TIMEOUT);
}

int splitkv_read_cta_times(const splitkv_plan_t* plan, int which, int64_t* out_ns, int64_t capacity,
                           void* stream) {
  if (!plan || !out_ns) return SPLITKV_ERR_INVALID_ARG;
  const DevPlan* dp = splitkv::plan_device_view(plan);
  if (!dp) return SPLITKV_ERR_NOT_UPLOADED;
  if (which != SPLITKV_WS_FWD && which != SPLITKV_WS_BWD && which != SPLITKV_TIMES_DQ) return SPLITKV_ERR_INVALID_ARG;
  // stamps: forward CTAs, then dK/dV CTAs, then dQ CTAs
  const int n = which == SPLITKV_WS_BWD ? dp->Wb : dp->W;
  if (capacity < n) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;
  const size_t first = which == SPLITKV_WS_FWD ? 0 : which == SPLITKV_WS_BWD ? size_t(dp->W) : size_t(dp->W + dp->Wb);
  const long long* src = dp->timers + 2 * first;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // stamps are small: copy to a host array synchronously on the stream
  long long* host = new (std::nothrow) long long[2 * size_t(n)];
  if (!host) return SPLITKV_ERR_NO_MEMORY;
  int st = cuda_status(cudaMemcpyAsync(host, src, 2 * size_t(n) * sizeof(long long), cudaMemcpyDeviceToHost, s));
  if (st == SPLITKV_OK) st = cuda_status(cudaStreamSynchronize(s));
  if (st == SPLITKV_OK)
    for (int i = 0; i < n; ++i) out_ns[i] = host[2 * i + 1] - host[2 * i];
  delete[] host;
  return st;
}

}  // extern "C"
