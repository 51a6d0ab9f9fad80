// Internal declarations shared by the host planner, the C-ABI layer and the
// sm_100a kernels of libsplitkv.so.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "splitkv.h"

namespace splitkv {

// Rows of one query tile: 128 / (G * bs) blocks x G heads x bs tokens.
constexpr int kTileRows = 128;

// Device view of a plan.  Every table lives in one device allocation owned by
// the plan; this struct is passed by value as a kernel parameter.
struct DevPlan {
  const int4* entries;          // [E]   {block, lo, hi, chunk}, record order
  const int4* tiles;            // [T]   {e0, e1, klo, khi}: entries [e0, e1), key union [klo, khi)
  const int4* fwd_items;        // [If]  {chunk, kv head, t0, t1} grouped by worker
  const int*  fwd_worker_ptr;   // [W+1]
  const int4* bwd_items;        // [Ib]  same, backward schedule (whole chunks)
  const int*  bwd_worker_ptr;   // [W+1]
  const int*  block_entry_ptr;  // [A+1]
  const int*  block_entries;    // [E]   entry ids of each block, ascending chunk
  const int*  zero_chunks;      // [Z]   chunks no block reads (backward zero fill)
  long long*  timers;           // [2W + Wb][2] global-timer stamps: forward, dK/dV, then dQ CTAs
  int*        status;           // device status word: 0, or a SPLITKV_ERR_* code a kernel recorded
  int num_zero_chunks;
  int N, Nq, A, bs, Hq, Hkv, G, d, C, num_chunks, E, W, Wb;
  int block_term;               // 1: separate block keys kb, vb (reading A); 0: block keys in the context
  int bt_lo, bt_hi;             // blocks [bt_lo, bt_hi) take the in-block term (all of them, but on a rank's shard)
  int partial_bf16;             // 1: O_c records and dQ partials stored as bf16
  // run-time claims (SPLITKV_FLAG_DYNAMIC_CLAIM): fwd_items / bwd_items hold the whole
  // lists in LPT order and the CTAs claim them through claim[0] (forward kernel),
  // claim[1] (dK/dV kernel), claim[2] (dQ kernel), zeroed before each launch
  int dynamic;
  int n_fwd_items, n_bwd_items;
  int* claim;                   // [4]
  // time limit of the kernels' mbarrier waits (ns; splitkv_plan_set_wait_limit), after
  // which a wait records SPLITKV_ERR_TIMEOUT and the kernel winds down
  long long wait_limit_ns;
};

// Byte offsets of the forward workspace (partial records).
struct FwdWs {
  size_t o_off, m_off, l_off, total;
};
// Byte offsets of the backward workspace (dq partials, Delta).
struct BwdWs {
  size_t dq_off, delta_off, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// rec_bytes: bytes of one O_c / dQ-partial element (4, or 2 under bf16 partials)
inline FwdWs fwd_ws_layout(long long E, int bs, int Hq, int d, size_t rec_bytes) {
  FwdWs w;
  const size_t rows = size_t(E) * bs * Hq;
  w.o_off = 0;
  w.m_off = align_up(rows * d * rec_bytes, 256);
  w.l_off = w.m_off + align_up(rows * sizeof(float), 256);
  w.total = w.l_off + align_up(rows * sizeof(float), 256);
  if (w.total == 0) w.total = 256;
  return w;
}

inline BwdWs bwd_ws_layout(long long E, int Nq, int bs, int Hq, int d, size_t rec_bytes) {
  BwdWs w;
  const size_t rows = size_t(E) * bs * Hq;
  w.dq_off = 0;
  w.delta_off = align_up(rows * d * rec_bytes, 256);
  w.total = w.delta_off + align_up(size_t(Nq) * Hq * sizeof(float), 256);
  return w;
}

// ---- TMA tensor maps (tensor_maps.cpp) ------------------------------------
// 3-D bf16 tensor [dim2][dim1][dim0] (dim0 contiguous), box {64, box1, box2},
// 128-byte swizzle, zero fill out of bounds; `map` points at a CUtensorMap.
bool tensor_maps_available();
bool make_bf16_map_3d(void* map, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box1,
                      uint32_t box2);
// 3-D fp32 tensor [dim2][dim1][dim0], box {box0, box1, box2}; box0 * 4 is 64
// or 128 bytes and selects the 64- or 128-byte swizzle (bulk stores of
// epilogue chunks).
bool make_f32_map_3d(void* map, void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box0,
                     uint32_t box1, uint32_t box2);
// 3-D bf16 tensor [dim2][dim1][dim0], box {32, box1, box2} (64-byte rows),
// 64-byte swizzle (bulk stores of bf16 epilogue chunks).
bool make_bf16_store_map_3d(void* map, void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2, uint32_t box1,
                            uint32_t box2);

// ---- kernel launchers (defined in the .cu files) ---------------------------
// part_o / dq_part: float32 records, or bf16 when p.partial_bf16 (tcgen05 path only)
cudaError_t launch_fwd_partial(const DevPlan& p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, float scale, void* part_o, float* part_m,
                               float* part_l, cudaStream_t s);

// Where the merge writes its rows.  o == nullptr: the plan's own outputs (o, lse, every
// query row).  Otherwise the exchange of Split-KV over ranks fused into the merge: the
// rows of block b go to the receive buffers of the rank that owns b (blocks
// [floor(r A / R), floor((r + 1) A / R)) to rank r) -- o[r] float32 [R][rows_r][Hq][d],
// lse[r] [R][rows_r][Hq] -- at slot `self`; o and lse are device arrays of R pointers,
// which may point into other GPUs' memory (peer-mapped).  The dQ reduce uses o for its dq
// rows (same layout) and ignores lse.
struct MergeDest {
  float* const* o;
  float* const* lse;
  int R, self;
};

cudaError_t launch_merge(const DevPlan& p, const uint16_t* q, const uint16_t* kb,
                         const uint16_t* vb, float scale, const void* part_o,
                         const float* part_m, const float* part_l, void* o, int o_bf16,
                         float* lse, cudaStream_t s, const MergeDest& dest = MergeDest{nullptr, nullptr, 1, 0});

// R and rank of a plan (1 and 0 unless made by splitkv_plan_shard).
void plan_ranks(const splitkv_plan_t* plan, int* R, int* rank);

cudaError_t launch_bwd_delta(const DevPlan& p, const void* o, int o_bf16, const uint16_t* dout,
                             float* delta, cudaStream_t s);

// which: 0 = both parts, 1 = the dK/dV part (everything on the mma.sync path),
// 2 = the dQ part (nothing on the mma.sync path).
cudaError_t launch_bwd_partial(const DevPlan& p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const uint16_t* dout, const float* lse,
                               const float* delta, float scale, float* dk, float* dv,
                               void* dq_part, cudaStream_t s, int which = 0);

cudaError_t launch_bwd_reduce(const DevPlan& p, const uint16_t* q, const uint16_t* kb,
                              const uint16_t* vb, const uint16_t* dout, const float* lse,
                              const float* delta, const void* dq_part, float scale, float* dq,
                              float* dkb, float* dvb, cudaStream_t s,
                              const MergeDest& dest = MergeDest{nullptr, nullptr, 1, 0});

// ---- argument checks shared by the C-ABI entry points (api.cpp, static_scratch.cu)
const DevPlan* plan_device_view(const splitkv_plan_t* P);

inline bool ptr_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Non-null and 16-byte aligned, every one of them.
template <typename... Ps>
inline bool all_aligned16(Ps... ps) {
  return ((ps != nullptr && ptr_aligned(ps, 16)) && ...);
}

// Block-key tensors (kb, vb, dkb, dvb): required under reading A; under reading B
// they may be NULL (never read or written) and are checked only for alignment.
template <typename... Ps>
inline bool block_ptrs_ok(const DevPlan* dp, Ps... ps) {
  if (dp->block_term) return all_aligned16(ps...);
  return ((ps == nullptr || ptr_aligned(ps, 16)) && ...);
}

// Bytes of one O_c / dQ-partial element of the plan's records.
inline size_t rec_bytes(const DevPlan* dp) { return dp->partial_bf16 ? 2 : 4; }

// True when the tcgen05 forward and backward kernels serve this plan (and no
// SPLITKV_FWD_KERNEL / SPLITKV_BWD_KERNEL override selects mma.sync): bf16
// partial records and run-time claims exist on those kernels only.
bool tcgen05_supported(const DevPlan& p);

// Checks every attention call shares; on success *out points at the plan's device view.
inline int check_plan(const splitkv_plan_t* plan, const DevPlan** out) {
  if (!plan) return SPLITKV_ERR_INVALID_ARG;
  const DevPlan* dp = plan_device_view(plan);
  if (!dp) return SPLITKV_ERR_NOT_UPLOADED;
  if (dp->d != 64 && dp->d != 128) return SPLITKV_ERR_UNSUPPORTED;
  if ((dp->partial_bf16 || dp->dynamic) && !tcgen05_supported(*dp)) return SPLITKV_ERR_UNSUPPORTED;
  *out = dp;
  return SPLITKV_OK;
}

}  // namespace splitkv
