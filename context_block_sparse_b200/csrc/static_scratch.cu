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
// the process exits.  In host code `g_scratch` names a host-side stand-in, not
// the device array, so its device address is looked up with
// cudaGetSymbolAddress.  That address belongs to the CUDA context the lookup
// ran in (a caller may make its own driver-API context current, and a context
// that is destroyed and re-created may load the module elsewhere), so the
// lookups are cached by the context's process-unique id (cuCtxGetId), not by
// device ordinal: in the ordinary case of one primary context per device that
// is one lookup per device.
#include <cstdint>
#include <mutex>

#include <cuda.h>

#include "splitkv.h"
#include "splitkv_internal.h"

namespace {

constexpr size_t kScratchBytes = SPLITKV_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Driver entry points, looked up through the runtime (no link-time libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(ptr);
  cudaGetLastError();
  return nullptr;
}

// Id of the context current on this thread; 0 when there is none yet.
int current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return SPLITKV_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return SPLITKV_ERR_CUDA;
  *id = 0;
  if (ctx != nullptr && get_id(ctx, id) != CUDA_SUCCESS) return SPLITKV_ERR_CUDA;
  return SPLITKV_OK;
}

constexpr int kCacheSlots = 64;
std::mutex g_scratch_mu;
unsigned long long g_ctx_id[kCacheSlots] = {};
void* g_ctx_addr[kCacheSlots] = {};
int g_slots_used = 0;

// Device address of g_scratch in the context current on this thread.  The first
// call in a context looks it up (which also initialises the device's primary
// context when the thread has none yet); later calls in the same context read
// the cache.  When more than kCacheSlots contexts have been seen, the extra ones
// look the address up on every call.
int scratch_address(void** out) {
  unsigned long long id = 0;
  int st = current_context_id(&id);
  if (st != SPLITKV_OK) return st;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (id != 0) {
    for (int i = 0; i < g_slots_used; ++i)
      if (g_ctx_id[i] == id) {
        *out = g_ctx_addr[i];
        return SPLITKV_OK;
      }
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return SPLITKV_ERR_CUDA;
  }
  if (id == 0 && (st = current_context_id(&id)) != SPLITKV_OK) return st;   // the lookup made one current
  if (id != 0 && g_slots_used < kCacheSlots) {
    g_ctx_id[g_slots_used] = id;
    g_ctx_addr[g_slots_used] = p;
    ++g_slots_used;
  }
  *out = p;
  return SPLITKV_OK;
}

}  // namespace

extern "C" int splitkv_attn_fwd_static_scratch(const splitkv_plan_t* plan, const void* q, const void* k,
                                               const void* v, const void* kb, const void* vb, float scale,
                                               void* o, int o_dtype, float* lse, void* stream) {
  // the same argument checks as splitkv_attn_fwd + splitkv_merge
  const splitkv::DevPlan* dp = nullptr;
  int st = splitkv::check_plan(plan, &dp);
  if (st != SPLITKV_OK) return st;
  if (!splitkv::all_aligned16(q, k, v, o) || !splitkv::block_ptrs_ok(dp, kb, vb) || !lse ||
      !splitkv::ptr_aligned(lse, 4))
    return SPLITKV_ERR_INVALID_ARG;
  if (o_dtype != SPLITKV_DTYPE_F32 && o_dtype != SPLITKV_DTYPE_BF16) return SPLITKV_ERR_INVALID_ARG;
  const splitkv::FwdWs L = splitkv::fwd_ws_layout(dp->E, dp->bs, dp->Hq, dp->d, splitkv::rec_bytes(dp));
  if (L.total > kScratchBytes) return SPLITKV_ERR_WORKSPACE_TOO_SMALL;   // problem too large for the buffer
  void* base = nullptr;
  st = scratch_address(&base);
  if (st != SPLITKV_OK) return st;
  char* w = static_cast<char*>(base);
  void* po = w + L.o_off;
  float* pm = reinterpret_cast<float*>(w + L.m_off);
  float* pl = reinterpret_cast<float*>(w + L.l_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Every record the merge reads is written by the partial kernel of the same
  // call, so nothing left over from an earlier call is read and nothing needs
  // clearing first.  (Run-time claims reset their cursor, which lives in the
  // plan's device memory, before the launch.)
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
