// sm_100a (Blackwell) primitives used by the tcgen05 kernels: mbarriers with
// bounded waits, TMA tensor loads, tensor-memory allocation, UMMA descriptors,
// tcgen05.mma / commit / ld / st.  Written from the public PTX ISA.
#pragma once

#include <cstdint>

#include <cuda.h>

#include "common.cuh"

namespace splitkv {
namespace sm100 {

// A wait that has not completed after this long has failed (a bug): the
// kernel records a timeout and the waiting site in its status words and winds
// down instead of hanging the GPU.  Bounded in time, not in iterations, because
// mbarrier.try_wait may suspend the thread between polls.  The kernels' ordinary
// waits take the plan's limit (this by default; a test may shorten it to make a
// wait run out); the drains of copies and products in flight on the way out
// always take this one, so that nothing is left writing after the CTA exits.
constexpr long long kWaitLimitNs = 2000000000LL;

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// One arrival per warp: the warp barrier orders every lane's earlier work (its
// tcgen05 operations, fenced with tc_fence_before, and its shared-memory
// accesses) before lane 0's release-arrive.  Barriers signalled this way count
// warps, not threads.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Where waits report: abort_flag (shared memory) makes every role of the CTA
// wind down; status (global, two words) receives the error code and the site
// of the first wait that timed out.
struct WaitCtx {
  volatile int* abort_flag;
  int* status;
  long long limit_ns;   // time limit of mbar_wait / warp_wait
};

__device__ __forceinline__ void record_timeout(const WaitCtx& c, int site) {
  *c.abort_flag = 1;
  atomicCAS(c.status + 1, 0, site);
  atomicExch(c.status, -5);   // SPLITKV_ERR_TIMEOUT
}

// Wait for the phase of `parity` to complete.  Returns false when the time
// limit passes (recorded with `site`) or another role has flagged an abort.  The
// clock is read every 64 polls, or at every poll under a limit below 1 us (a
// limit of 0 gives up at the first poll that finds the phase incomplete).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& c, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0 || c.limit_ns < 1000) {
      if (*c.abort_flag) return false;
      if (global_timer_ns() - t0 >= c.limit_ns) {
        record_timeout(c, site);
        return false;
      }
    }
  }
}

// Every lane of the warp waits (each gets the acquire), and the outcome is made
// warp-uniform so that the warp-collective tcgen05 operations that follow are
// executed by all lanes or by none.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& c, int site) {
  const bool ok = mbar_wait(bar, parity, c, site);
  return __all_sync(0xffffffffu, ok) != 0;
}

// Bounded wait that ignores the abort flag (drains copies or MMAs in flight).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, const WaitCtx& c, int site) {
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
      record_timeout(c, site);
      return;
    }
  }
}

// ---------------------------------------------------------------- run-time item claims
// Items claimed at run time: whenever the producer thread of a CTA needs a new
// item it takes the next index of a global cursor (one atomicAdd) and hands it
// to the CTA's other roles through a ring of shared-memory slots, so that every
// role walks the same sequence; an index past the list ends it (-1 in the ring).
// A CTA therefore takes the next item of the list as soon as it is free: the
// list order (longest first) with the actual, not the predicted, loads.
constexpr int kClaimRing = 4;
struct ClaimRing {
  uint64_t full[kClaimRing];    // count 1: the producer's arrival after it wrote the slot
  uint64_t empty[kClaimRing];   // count: the consumers' arrivals (threads or warps)
  int item[kClaimRing];
};
// Thread 0, before the CTA's mbarrier-init fence.
__device__ __forceinline__ void claim_ring_init(ClaimRing* r, uint32_t consumers) {
  for (int s = 0; s < kClaimRing; ++s) {
    mbar_init(&r->full[s], 1);
    mbar_init(&r->empty[s], consumers);
  }
}

enum ClaimRole { kClaimProducer = 0, kClaimThread = 1, kClaimWarp = 2 };

// The item sequence one role of a CTA walks: a static range [it, end) of the
// schedule's item list, or (cursor != nullptr) the run-time claims over the
// whole list of `end` items.  A kClaimWarp role calls next() with all 32 lanes.
struct ItemSeq {
  ClaimRing* ring;
  int* cursor;
  int it, end;
  uint32_t cnt;
  int role;
  __device__ void init_static(int first, int last) {
    ring = nullptr;
    cursor = nullptr;
    it = first;
    end = last;
    cnt = 0;
    role = kClaimThread;
  }
  __device__ void init_claims(ClaimRing* r, int* cur, int n_items, int role_) {
    ring = r;
    cursor = cur;
    it = 0;
    end = n_items;
    cnt = 0;
    role = role_;
  }
  // The next item index; false at the end of the sequence, or when a wait gave up
  // (the wait recorded the timeout, or another role's abort stopped it).
  __device__ bool next(int& idx, const WaitCtx& c, int site) {
    if (cursor == nullptr) {
      if (it >= end) return false;
      idx = it++;
      return true;
    }
    const int s = int(cnt % kClaimRing);
    const uint32_t ph = (cnt / kClaimRing) & 1u;
    ++cnt;
    int v;
    if (role == kClaimProducer) {
      // the slot is free once every consumer took the item it held kClaimRing claims ago
      if (!mbar_wait(&ring->empty[s], ph ^ 1u, c, site)) return false;
      v = atomicAdd(cursor, 1);
      if (v >= end) v = -1;
      ring->item[s] = v;
      mbar_arrive(&ring->full[s]);   // release: the slot's write before the arrival
    } else if (role == kClaimThread) {
      if (!mbar_wait(&ring->full[s], ph, c, site)) return false;
      v = *reinterpret_cast<volatile int*>(&ring->item[s]);
      mbar_arrive(&ring->empty[s]);
    } else {
      if (!warp_wait(&ring->full[s], ph, c, site)) return false;
      v = *reinterpret_cast<volatile int*>(&ring->item[s]);
      warp_arrive(&ring->empty[s]);
    }
    if (v < 0) return false;
    idx = v;
    return true;
  }
};

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Bulk tensor store shared -> global (bulk-group completion) and its waits.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One warp's 32 rows x 16 fp32 columns (vals[0..16) of the lane's row, times
// mul) through a 2 KB shared buffer laid out as the 64-byte-swizzled box of
// `map` (row = lane), then one bulk tensor store at (x, y, z) when `store`.
// Before the buffer is rewritten, at most kPending of this lane-0's earlier bulk
// stores may still be reading shared memory: 1 for a warp alternating two
// buffers, 0 for a warp with one.  The buffer must be 512-byte aligned; lane 0
// owns the bulk groups (bulk_wait0 before the CTA exits).
template <int kPending>
__device__ __forceinline__ void warp_bulk_store16(float* buf, const uint32_t* vals, float mul,
                                                  const CUtensorMap* map, int x, int y, int z, bool store = true) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kPending) : "memory");
  __syncwarp();
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float4 v = make_float4(__uint_as_float(vals[4 * g]) * mul, __uint_as_float(vals[4 * g + 1]) * mul,
                                 __uint_as_float(vals[4 * g + 2]) * mul, __uint_as_float(vals[4 * g + 3]) * mul);
    *reinterpret_cast<float4*>(buf + lane * 16 + ((g ^ ((lane >> 1) & 3)) << 2)) = v;
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0 && store) {
    tma_store_3d(map, buf, x, y, z);
    bulk_commit();
  }
  __syncwarp();
}

// The bf16 counterpart: one warp's 32 rows x 32 columns (vals[0..32) of the
// lane's row, times mul, rounded to bf16 with round-to-nearest-even) through a
// 2 KB buffer laid out as the 64-byte-swizzled box {32, ...} of a bf16 `map`,
// then one bulk tensor store at (x, y, z) when `store`.  Same buffer rules as
// warp_bulk_store16.
template <int kPending>
__device__ __forceinline__ void warp_bulk_store32_bf16(float* bufp, const uint32_t* vals, float mul,
                                                       const CUtensorMap* map, int x, int y, int z, bool store = true) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kPending) : "memory");
  __syncwarp();
  uint32_t* buf = reinterpret_cast<uint32_t*>(bufp);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint4 w;
    w.x = pack_bf16(__uint_as_float(vals[8 * g]) * mul, __uint_as_float(vals[8 * g + 1]) * mul);
    w.y = pack_bf16(__uint_as_float(vals[8 * g + 2]) * mul, __uint_as_float(vals[8 * g + 3]) * mul);
    w.z = pack_bf16(__uint_as_float(vals[8 * g + 4]) * mul, __uint_as_float(vals[8 * g + 5]) * mul);
    w.w = pack_bf16(__uint_as_float(vals[8 * g + 6]) * mul, __uint_as_float(vals[8 * g + 7]) * mul);
    *reinterpret_cast<uint4*>(buf + lane * 16 + ((g ^ ((lane >> 1) & 3)) << 2)) = w;
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0 && store) {
    tma_store_3d(map, buf, x, y, z);
    bulk_commit();
  }
  __syncwarp();
}

// 32 values of the lane's own row, times mul, as bf16 to dst (64 bytes, 16-byte
// aligned): four 16-byte stores (rows that are not one bulk box).
__device__ __forceinline__ void lane_store32_bf16(uint16_t* dst, const uint32_t* vals, float mul) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint4 w;
    w.x = pack_bf16(__uint_as_float(vals[8 * g]) * mul, __uint_as_float(vals[8 * g + 1]) * mul);
    w.y = pack_bf16(__uint_as_float(vals[8 * g + 2]) * mul, __uint_as_float(vals[8 * g + 3]) * mul);
    w.z = pack_bf16(__uint_as_float(vals[8 * g + 4]) * mul, __uint_as_float(vals[8 * g + 5]) * mul);
    w.w = pack_bf16(__uint_as_float(vals[8 * g + 6]) * mul, __uint_as_float(vals[8 * g + 7]) * mul);
    reinterpret_cast<uint4*>(dst)[g] = w;
  }
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- UMMA
// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;   // version
  d |= uint64_t(2) << 61;   // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator,
// A K-major, B K-major (b_mn_major = 0) or MN-major (1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int b_mn_major) {
  return (1u << 4)                      // D format f32
         | (1u << 7)                    // A format bf16
         | (1u << 10)                   // B format bf16
         | (uint32_t(b_mn_major) << 16) // B major
         | (uint32_t(N >> 3) << 17)     // N / 8
         | (uint32_t(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- TMEM <-> registers
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// tcgen05.ld writes its destination registers asynchronously: after
// tmem_wait_ld, pass the loaded values through this empty asm so that the
// compiler cannot move any use of them above the wait.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t* r) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// Same, into r[0..32) of a larger register array (unrolled by the caller).
__device__ __forceinline__ void tmem_ld32p(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16p(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 16-lane shapes (a warp reads or writes 16 TMEM lanes starting at the lane of
// taddr, inside its own quarter).  Register fragments, measured on the B200: in
// every repetition i of 16x256b (8 columns wide), thread t holds lanes t/4 and
// t/4 + 8 (relative to the first lane), columns 8i + 2(t % 4) and + 1, as
// r[4i .. 4i+3] = (t/4, c), (t/4, c+1), (t/4+8, c), (t/4+8, c+1); in repetition i
// of 16x128b (4 columns wide), r[2i] is lane t/4 and r[2i+1] lane t/4 + 8, both
// at column 4i + t % 4.  So the bf16 pair of the two adjacent fp32 columns a
// thread loads with 16x256b goes back with 16x128b to one 32-bit column of the
// same lane: the packed layout the MMA reads P from.
__device__ __forceinline__ void tmem_ld16x256b_x16(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16x128b_x8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16x256b_x4(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16x256b_x4(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Paired fp32 arithmetic (two lanes of work per instruction).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- exp2 on the FMA pipe
// 2^x for two lanes without the MUFU unit (which computes only 16 exp2 per
// clock per SM): Cody-Waite range reduction x = n + f, n = round(x) (by adding
// and subtracting 1.5 * 2^23), f in [-0.5, 0.5], a cubic fitted here to 2^f on
// that interval (weighted least squares on the relative error, max relative
// error 7.6e-5 in fp32, far below bf16's 3.9e-3), and the exponent n added
// to the result's bits.  Below -126 (and for -inf, a masked score) the result
// is exactly 0, as MUFU's is for -inf.
constexpr float kExpMagic = 12582912.0f;   // 1.5 * 2^23
constexpr float kExpC0 = 0.99992758f, kExpC1 = 0.69326109f, kExpC2 = 0.24261758f, kExpC3 = 0.055174146f;

__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  const bool z0 = x0 < -126.f, z1 = x1 < -126.f;
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0, t1, n0, n1, f0, f1, p0, p1;
  fadd2(t0, t1, x0, x1, kExpMagic, kExpMagic);     // round(x) in the low mantissa bits
  fadd2(n0, n1, t0, t1, -kExpMagic, -kExpMagic);   // round(x) as a float
  fadd2(f0, f1, x0, x1, -n0, -n1);                 // f = x - n
  ffma2(p0, p1, f0, f1, kExpC3, kExpC3, kExpC2, kExpC2);
  ffma2(p0, p1, p0, p1, f0, f1, kExpC1, kExpC1);
  ffma2(p0, p1, p0, p1, f0, f1, kExpC0, kExpC0);
  y0 = z0 ? 0.f : __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = z1 ? 0.f : __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// exp2 of two lanes on MUFU (poly = false) or on the FMA pipe (poly = true);
// callers pass a condition on an unrolled loop index, so the branch folds away.
__device__ __forceinline__ void exp2_pair(bool poly, float x0, float x1, float& y0, float& y1) {
  if (poly) {
    exp2_poly2(x0, x1, y0, y1);
  } else {
    y0 = fast_exp2(x0);
    y1 = fast_exp2(x1);
  }
}

// One pair in kPolyEvery goes through the polynomial (keeps MUFU and FMA busy).
constexpr int kPolyEvery = 4;

// ---------------------------------------------------------------- epilogue stores
// Lane i of a warp holds W consecutive fp32 values of its own output row
// (vals[0..W)); dst is that row's destination (NULL for a row that is not
// written).  The values go through a per-warp scratch of 32 x W floats in
// shared memory so that every global store instruction writes whole 4W-byte
// row segments of 128 / W rows instead of 32 scattered 16-byte pieces.
// W is 16 or 32; the scratch is XOR-swizzled by 16-byte granule.
template <int W>
__device__ __forceinline__ void warp_store_rows(float* scratch, const float* vals, float mul, float* dst) {
  constexpr int kG = W / 4;          // 16-byte granules per row
  constexpr int kRows = 32 / kG;     // rows per store instruction
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int g = 0; g < kG; ++g) {
    const float4 x = make_float4(vals[4 * g] * mul, vals[4 * g + 1] * mul, vals[4 * g + 2] * mul,
                                 vals[4 * g + 3] * mul);
    *reinterpret_cast<float4*>(scratch + lane * W + ((g ^ (lane & (kG - 1))) << 2)) = x;
  }
  __syncwarp();
  const unsigned long long mine = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
  for (int k = 0; k < kG; ++k) {
    const int r = k * kRows + lane / kG;
    const int gi = lane % kG;
    const float4 x = *reinterpret_cast<const float4*>(scratch + r * W + ((gi ^ (r & (kG - 1))) << 2));
    float* d = reinterpret_cast<float*>(__shfl_sync(0xffffffffu, mine, r));
    if (d != nullptr) *reinterpret_cast<float4*>(d + 4 * gi) = x;
  }
  __syncwarp();
}

}  // namespace sm100
}  // namespace splitkv
