// Forward attention whose partial records live in a library-owned, statically
// sized device buffer, so that a call allocates no device memory.
//
// Who needs this: callers that may not call cudaMalloc on their hot path --
// code running inside a framework whose caching allocator has reserved the
// device memory (a cudaMalloc there fails or forces the framework to release
// its cache), real-time or latency-critical loops where cudaMalloc's implicit
// device synchronisation is not acceptable, and plug-in code that is handed
// raw pointers but no allocator.  They build and upload a plan once at set-up
// (splitkv_plan_upload is the only allocating step) and afterwards call this
// entry point with their own input and output buffers only.
//
// The scratch array below is part of the module image: every GPU that loads
// this library holds SPLITKV_STATIC_SCRATCH_BYTES of device memory for it until
// the process exits.  Its device address is looked up once per device.
#include <cstdint>
#include <mutex>

#include "splitkv.h"
#include "splitkv_internal.h"

namespace splitkv {
const DevPlan* plan_device_view(const splitkv_plan_t* P);
}

namespace {

constexpr size_t kScratchBytes = SPLITKV_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up on first use).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SPLITKV_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SPLITKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SPLITKV_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SPLITKV_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

}  // namespace

extern "C" int splitkv_attn_fwd_static_scratch(const splitkv_plan_t* plan, const void* q, const void* k,
                                               const void* v, const void* kb, const void* vb, float scale,
                                               void* o, int o_dtype, float* lse, void* stream) {
  if (!plan) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::DevPlan* dp = splitkv::plan_device_view(plan);
  if (!dp) return SPLITKV_ERR_NOT_UPLOADED;
  if (dp->d != 64 && dp->d != 128) return SPLITKV_ERR_UNSUPPORTED;
  if ((dp->partial_bf16 || dp->dynamic) && !splitkv::tcgen05_supported(*dp)) return SPLITKV_ERR_UNSUPPORTED;
  // kb, vb: required under reading A; may be NULL under SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT
  const bool blk_ok = dp->block_term ? (aligned16(kb) && aligned16(vb))
                                     : ((!kb || aligned16(kb)) && (!vb || aligned16(vb)));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !blk_ok || !aligned16(o) || !lse ||
      (reinterpret_cast<uintptr_t>(lse) % 4) != 0)
    return SPLITKV_ERR_INVALID_ARG;
  if (o_dtype != SPLITKV_DTYPE_F32 && o_dtype != SPLITKV_DTYPE_BF16) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::FwdWs L = splitkv::fwd_ws_layout(dp->E, dp->bs, dp->Hq, dp->d, dp->partial_bf16 ? 2 : 4);
  if (L.total > kScratchBytes) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;   // problem too large for the buffer
  void* base = nullptr;
  const int st = scratch_address(&base);
  if (st != SPLITKV_OK) return st;
  char* w = static_cast<char*>(base);
  void* po = w + L.o_off;
  float* pm = reinterpret_cast<float*>(w + L.m_off);
  float* pl = reinterpret_cast<float*>(w + L.l_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Every record the merge reads is written by the partial kernel of the same
  // call, so nothing left over from an earlier call is read.
  cudaError_t e = splitkv::launch_fwd_partial(*dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                              static_cast<const uint16_t*>(v), scale, po, pm, pl, s);
  if (e == cudaSuccess)
    e = splitkv::launch_merge(*dp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kb),
                              static_cast<const uint16_t*>(vb), scale, po, pm, pl, o,
                              o_dtype == SPLITKV_DTYPE_BF16 ? 1 : 0, lse, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SPLITKV_ERR_CUDA;
  }
  return SPLITKV_OK;
}
