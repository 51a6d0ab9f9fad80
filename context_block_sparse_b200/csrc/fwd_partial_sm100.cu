// Partial attention of every (chunk, block) entry on the 5th-generation tensor
// cores (tcgen05 / TMEM / TMA), head_dim 64 or 128.
//
// News page "Split-KV speeds diffusion drafter training by keeping long-context
// data local", section "Exchange the smaller side": each key/value shard (here
// a KV chunk) evaluates every query that reads it and emits a partial result
// with its normalisation statistics; section "Balance actual attention work":
// the shards are spread over workers (here persistent CTAs) by LPT.
//
// One persistent CTA per worker walks its LPT items; every item's 128-row query
// tiles are taken two at a time (A and B) so that each K/V tile loaded into
// shared memory feeds two 128x128 score tiles.  Roles (512 threads):
//   warp 0      TMA producer: Q tiles (3-D boxes of bs tokens x G heads per
//               block) and 128-key K and V tiles into two-stage rings of their
//               own (a K stage refills once its S products are done, a V stage
//               once its PV products are; a pair's first K/V tiles go out before
//               its Q buffer frees);
//   warp 1      MMA issuer (one thread): S_X = Q_X K^T into TMEM, then
//               O_X += P_X V with P_X read from TMEM (bf16, aliasing S_X);
//   warp 2      tensor-memory allocation (512 columns: S_A, S_B, O_A, O_B);
//   warps 4-11  softmax of both tiles (A, then B, at every key tile): warp 4 + q
//               holds rows 32q..32q+15 and warp 8 + q rows 32q+16..32q+31 through
//               the 16-lane TMEM shapes, two rows and 32 columns per thread, so
//               that the four threads of a row reduce its maximum by shuffles;
//   warps 12-15 record epilogue of both tiles: O_X / l from TMEM to the record,
//               so that the softmax warps go on to the next pair at once and the
//               output columns return to the MMA right after their last read.
// The softmax keeps, per row, a reference maximum m_ref, taken from the first
// key tile in which the row has allowed keys; later tiles exponentiate against
// it, and only when a score exceeds m_ref by more than 2^32 (in P) are O and l
// rescaled to a new reference -- the result is the same, the reference is exact
// bookkeeping.  The record written is m_c = the row's true maximum (natural
// units), l_c = sum exp(s - m_c) and O_c = sum exp(s - m_c) v / l_c.
// Rows are masked to their block's [lo, hi).  The epilogue stores go through a
// 4 KB per-warp staging buffer so that every store instruction writes whole
// 128-byte row segments (bf16 records: 64 bytes per row straight from registers).
//
// Every mbarrier wait is bounded; on a timeout the kernel records
// SPLITKV_ERR_TIMEOUT in the plan's status word, lets every role wind down,
// waits for its own copies in flight and frees its tensor memory.
#include <cfloat>
#include <cstring>

#include "sm100.cuh"
#include "splitkv.h"
#include "splitkv_internal.h"

namespace splitkv {
namespace {

using namespace sm100;

constexpr int BM = 128;               // query rows per tile
constexpr int BN = 128;               // keys per key tile
constexpr int kStages = 2;            // K/V ring depth
constexpr int kThreads = 512;
constexpr uint32_t kHalf = 128 * 128; // bytes of one 64-column half of a 128-row tile
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
// A row's reference maximum stays while P = exp2(s - m_ref) <= 2^kHeadroomLog2;
// P (bf16), l and O (fp32) hold such values exactly as well as near 1, and
// O = sum P v stays far inside the fp32 range.
constexpr float kHeadroomLog2 = 32.0f;

// Sizes that follow the head dimension D (64 or 128): a 128-row bf16 tile of D
// columns is D / 64 halves of 16 KB, PV has N = D, O takes D TMEM columns.
// Shared-memory map (offsets from a 1024-aligned base).
template <int D>
struct Dims {
  static_assert(D == 64 || D == 128, "head dimension");
  static constexpr uint32_t kTile = uint32_t(D / 64) * kHalf;    // a 128 x D bf16 tile
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 1);
  static constexpr uint32_t kOffQ = 0;                              // Q_A, Q_B
  static constexpr uint32_t kOffK = kOffQ + 2 * kTile;              // K stages
  static constexpr uint32_t kOffV = kOffK + kStages * kTile;        // V stages
  static constexpr uint32_t kOffScratch = kOffV + kStages * kTile;  // record staging, 4 KB per epilogue warp
  static constexpr uint32_t kOffStats = kOffScratch + 4 * 4096;     // row statistics [2 pair parities][2 tiles][128] float4
  static constexpr uint32_t kOffRows = kOffStats + 2 * 2 * BM * 16; // allowed keys (lo, hi) [2 tiles][128] int2
  static constexpr uint32_t kOffBar = kOffRows + 2 * BM * 8;         // mbarriers
  static constexpr uint32_t kSmemBytes = kOffBar + 512 + 1024;      // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], v_full[kStages], k_empty[kStages], v_empty[kStages];
  uint64_t s_ready[2], p_ready[2], o_ready[2], o_free[2];
  // o_full[x]: tile x's last PV of a pair has completed (the epilogue reads O);
  // stats_ready[x][b]: the softmax warps of tile x left the row statistics of a pair
  // in stats buffer b = pair parity
  uint64_t o_full[2], stats_ready[2][2];
  uint64_t mma_done;
  ClaimRing ring;   // run-time claims: the producer hands items to the MMA thread and the 8 softmax warps
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");
constexpr uint32_t kClaimConsumers = 1 + 8 + 4;

// The sequence of tile pairs a worker processes (identical in every role): the
// worker's items of the static schedule, or the items it claims at run time.
struct PairIter {
  const DevPlan* p;
  const WaitCtx* wc;
  ItemSeq seq;      // item cursor
  int t, t_end;     // tile cursor inside the item
  int g;
  __device__ void init(const DevPlan* plan, int w, ClaimRing* ring, int role, const WaitCtx* wctx) {
    p = plan;
    wc = wctx;
    if (plan->dynamic)
      seq.init_claims(ring, plan->claim + 0, plan->n_fwd_items, role);
    else
      seq.init_static(plan->fwd_worker_ptr[w], plan->fwd_worker_ptr[w + 1]);
    t = t_end = 0;
    g = 0;
  }
  // tA, tB (-1 if absent), kv head, key union [klo, khi); false at the end (or
  // when a claim wait gave up, which the wait recorded)
  __device__ bool next(int& tA, int& tB, int& head, int& klo, int& khi) {
    while (t >= t_end) {
      int idx;
      if (!seq.next(idx, *wc, 1 * 10000 + __LINE__)) return false;
      const int4 item = p->fwd_items[idx];
      g = item.y;
      t = item.z;
      t_end = item.w;
    }
    tA = t++;
    tB = (t < t_end) ? t++ : -1;
    head = g;
    const int4 a = p->tiles[tA];
    klo = a.z;
    khi = a.w;
    if (tB >= 0) {
      const int4 b = p->tiles[tB];
      klo = min(klo, b.z);
      khi = max(khi, b.w);
    }
    return true;
  }
};


// The two rows a softmax thread holds in one query tile (16x256b fragments: rows
// t/4 and t/4 + 8 of its warp's 16 lanes): the reference maximum and the true
// maximum (log2 units), and the sum of P relative to the reference over this
// thread's 32 columns of each row (the four threads of a row add theirs at the
// end of the tile).  The rows' allowed keys live in shared memory.
struct Rows2 {
  float m_ref[2], m_true[2], l[2];
};

// Row maxima of the 64 scores a thread holds (32 per row; masked scores -inf),
// reduced over the four threads of each row.
__device__ __forceinline__ void row_max2(const uint32_t (&v)[64], float& m0, float& m1) {
  float a0 = -INFINITY, a1 = -INFINITY, b0 = -INFINITY, b1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    a0 = fmax3(a0, __uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]));
    b0 = fmax3(b0, __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    a1 = fmax3(a1, __uint_as_float(v[4 * i + 4]), __uint_as_float(v[4 * i + 5]));
    b1 = fmax3(b1, __uint_as_float(v[4 * i + 6]), __uint_as_float(v[4 * i + 7]));
  }
  m0 = fmaxf(a0, a1);
  m1 = fmaxf(b0, b1);
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
}

// P = exp2(v * c - m_row) for the thread's 64 scores (exactly 0 for a masked
// score, -inf), packed to bf16 pairs and stored with 16x128b over the scores'
// first 64 TMEM columns (P of keys 2k, 2k + 1 in column k); adds the rows' sums of
// the fp32 P to l0, l1.  MUFU for every exponential.
__device__ __forceinline__ void exp_pack_store2(const uint32_t (&v)[64], float c, float nm0, float nm1,
                                                uint32_t tS, float& l0, float& l1) {
  float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = 4 * (half * 8 + i);
      float x0, x1, y0, y1;
      ffma2(x0, x1, __uint_as_float(v[q]), __uint_as_float(v[q + 1]), c, c, nm0, nm0);
      ffma2(y0, y1, __uint_as_float(v[q + 2]), __uint_as_float(v[q + 3]), c, c, nm1, nm1);
      const float p0 = fast_exp2(x0), p1 = fast_exp2(x1), r0 = fast_exp2(y0), r1 = fast_exp2(y1);
      fadd2(s00, s01, s00, s01, p0, p1);
      fadd2(s10, s11, s10, s11, r0, r1);
      pk[2 * i] = pack_bf16(p0, p1);
      pk[2 * i + 1] = pack_bf16(r0, r1);
    }
    tmem_st16x128b_x8(tS + half * 32, pk);
  }
  l0 += s00 + s01;
  l1 += s10 + s11;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_partial_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, DevPlan p, float scale_log2,
                             void* __restrict__ part_o,
                             float* __restrict__ part_m, float* __restrict__ part_l) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using Dm = Dims<D>;
  constexpr uint32_t kTile = Dm::kTile;
  constexpr uint32_t kIdescPV = Dm::kIdescPV;
  constexpr uint32_t kOffQ = Dm::kOffQ, kOffK = Dm::kOffK, kOffV = Dm::kOffV;
  Bars* bars = reinterpret_cast<Bars*>(smem + Dm::kOffBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int w = blockIdx.x;
  volatile int* abort_flag = &bars->abort_flag;
  const WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};

  if (tid == 0) {
    p.timers[w * 2 + 0] = global_timer_ns();
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_ready[x], 1);
      mbar_init(&bars->p_ready[x], 8);    // one arrival per softmax warp
      mbar_init(&bars->o_ready[x], 1);
      mbar_init(&bars->o_free[x], 4);      // one arrival per epilogue warp
      mbar_init(&bars->o_full[x], 1);
      mbar_init(&bars->stats_ready[x][0], 8);
      mbar_init(&bars->stats_ready[x][1], 8);
    }
    mbar_init(&bars->mma_done, 1);
    claim_ring_init(&bars->ring, kClaimConsumers);
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int rows_per_slot = p.G * p.bs;
  const uint32_t slot_bytes = uint32_t(rows_per_slot) * 128;   // one slot's rows of one 64-column half
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      PairIter pi;
      pi.init(&p, w, &bars->ring, kClaimProducer, &wctx);
      int tA, tB, g, klo, khi;
      uint32_t kv_count = 0, pair_count = 0, q_issued = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      // key tile j of the current pair into the next K and V stages: each stage is
      // refilled once the last product reading it (S for K, PV for V) has completed
      auto load_kv = [&](int j) -> bool {
        const int s = kv_count % kStages;
        const uint32_t ph = ((kv_count / kStages) & 1) ^ 1;
        const int k0 = klo + j * BN;
        if (!mbar_wait(&bars->k_empty[s], ph, wctx, 1 * 10000 + __LINE__)) return false;
        mbar_expect_tx(&bars->k_full[s], kTile);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_3d(smem + kOffK + s * kTile + dh * kHalf, &tm_k, &bars->k_full[s], dh * 64, g, k0);
        ++k_issued;
        if (!mbar_wait(&bars->v_empty[s], ph, wctx, 1 * 10000 + __LINE__)) return false;
        mbar_expect_tx(&bars->v_full[s], kTile);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_3d(smem + kOffV + s * kTile + dh * kHalf, &tm_v, &bars->v_full[s], dh * 64, g, k0);
        ++v_issued;
        ++kv_count;
        return true;
      };
      while (ok && pi.next(tA, tB, g, klo, khi)) {
        const int n_kt = (khi - klo + BN - 1) / BN;
        // the pair's first K / V tiles go out before its Q buffer frees
        if (!load_kv(0)) { ok = false; break; }
        if (!mbar_wait(&bars->q_empty, (pair_count & 1) ^ 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
        const int4 ta = p.tiles[tA];
        const int nA = ta.y - ta.x;
        int nB = 0;
        int4 tb = make_int4(0, 0, 0, 0);
        if (tB >= 0) {
          tb = p.tiles[tB];
          nB = tb.y - tb.x;
        }
        // whole tiles: slots past a tile's last block come from token coordinate
        // Nq (outside the tensor) and are zero-filled
        const int nx = tB >= 0 ? 2 : 1;
        mbar_expect_tx(&bars->q_full, uint32_t(nx) * kTile);
        for (int x = 0; x < nx; ++x) {
          const int n = x == 0 ? nA : nB;
          const int e0 = x == 0 ? ta.x : tb.x;
          uint8_t* qbuf = smem + kOffQ + x * kTile;
          for (int s = 0; s < BM / rows_per_slot; ++s) {
            const int z = s < n ? p.entries[e0 + s].x * p.bs : p.Nq;
            for (int dh = 0; dh < D / 64; ++dh)
              tma_load_3d(qbuf + dh * kHalf + s * slot_bytes, &tm_q, &bars->q_full, dh * 64, g * p.G, z);
          }
        }
        ++q_issued;
        for (int j = 1; j < n_kt; ++j)
          if (!load_kv(j)) { ok = false; break; }
        if (!ok) break;
        ++pair_count;
      }
      if (!ok) *abort_flag = 1;
      // copies still in flight land before the CTA may exit: wait for the last
      // fill of every buffer (bounded; completed phases return at once)
      if (q_issued > 0) mbar_drain(&bars->q_full, (q_issued - 1) & 1, wctx, 1 * 10000 + __LINE__);
      for (uint32_t c = k_issued >= kStages ? k_issued - kStages : 0; c < k_issued; ++c)
        mbar_drain(&bars->k_full[c % kStages], (c / kStages) & 1, wctx, 1 * 10000 + __LINE__);
      for (uint32_t c = v_issued >= kStages ? v_issued - kStages : 0; c < v_issued; ++c)
        mbar_drain(&bars->v_full[c % kStages], (c / kStages) & 1, wctx, 1 * 10000 + __LINE__);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      PairIter pi;
      pi.init(&p, w, &bars->ring, kClaimThread, &wctx);
      int tA, tB, g, klo, khi;
      uint32_t kv_count = 0, pair_count = 0;
      uint32_t p_cnt[2] = {0, 0}, of_cnt[2] = {0, 0};
      bool ok = true;
      const uint32_t sQ = smem_u32(smem + kOffQ);
      const uint32_t sK = smem_u32(smem + kOffK);
      const uint32_t sV = smem_u32(smem + kOffV);
      while (ok && pi.next(tA, tB, g, klo, khi)) {
        const int nx = tB >= 0 ? 2 : 1;
        const int n_kt = (khi - klo + BN - 1) / BN;
        if (!mbar_wait(&bars->q_full, pair_count & 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
        {
          const int s0 = kv_count % kStages;
          if (!mbar_wait(&bars->k_full[s0], (kv_count / kStages) & 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
          tc_fence_after();
          for (int x = 0; x < nx; ++x) {
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t a = smem_desc_sw128(sQ + x * kTile + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
              const uint64_t b = smem_desc_sw128(sK + s0 * kTile + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
              mma_ss(tmem + x * 128, a, b, kIdescQK, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bars->s_ready[x]);
          }
          mma_commit(&bars->k_empty[s0]);   // K_s0 free once its S products complete
        }
        for (int j = 0; j < n_kt && ok; ++j) {
          const uint32_t c = kv_count + j;
          const int s = c % kStages;
          const int s1 = (c + 1) % kStages;
          const bool more = j + 1 < n_kt;
          for (int x = 0; x < nx; ++x) {
            if (!mbar_wait(&bars->p_ready[x], p_cnt[x] & 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
            ++p_cnt[x];
            if (j == 0) {
              if (!mbar_wait(&bars->o_free[x], (of_cnt[x] & 1) ^ 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
              ++of_cnt[x];
            }
            if (x == 0) {
              if (!mbar_wait(&bars->v_full[s], (c / kStages) & 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
            }
            tc_fence_after();
            // O_X (+)= P_X V : P in TMEM (keys 2k, 2k + 1 in column k of S_X), V MN-major
            // in smem
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint64_t b = smem_desc_sw128(sV + s * kTile + kk * 2048, kHalf, 1024);
              mma_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, b, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bars->o_ready[x]);
            if (!more) mma_commit(&bars->o_full[x]);           // tile x's output complete
            if (x == nx - 1) mma_commit(&bars->v_empty[s]);   // V_s: its last PV issued
            if (more) {
              if (x == 0) {
                if (!mbar_wait(&bars->k_full[s1], ((c + 1) / kStages) & 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
                tc_fence_after();
              }
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t a = smem_desc_sw128(sQ + x * kTile + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
                const uint64_t b =
                    smem_desc_sw128(sK + s1 * kTile + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
                mma_ss(tmem + x * 128, a, b, kIdescQK, kk > 0 ? 1u : 0u);
              }
              mma_commit(&bars->s_ready[x]);
              if (x == nx - 1) {
                mma_commit(&bars->k_empty[s1]);   // K_s1: its last S issued
                // the pair's last S: Q_A / Q_B have no further reader
                if (j + 2 == n_kt) mma_commit(&bars->q_empty);
              }
            }
          }
          if (!ok) break;
        }
        if (!ok) break;
        if (n_kt == 1) mma_commit(&bars->q_empty);
        kv_count += n_kt;
        ++pair_count;
      }
      if (!ok) *abort_flag = 1;
      // every MMA must finish before tensor memory is released
      mma_commit(&bars->mma_done);
      mbar_drain(&bars->mma_done, 0, wctx, 1 * 10000 + __LINE__);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ softmax
    // Warps 4-11 take both tiles of a pair, A then B at every key tile.  Warp 4 + q
    // holds rows 32q..32q+15 of a tile and warp 8 + q rows 32q+16..32q+31, through
    // the 16-lane TMEM shapes: each thread has two rows (t/4 and t/4 + 8 of its
    // warp's 16) and 32 of their 128 columns, the four threads of a row sit in one
    // warp and reduce its maximum with two shuffles.
    const int wq = warp & 3, h = (warp - 4) >> 2;
    const int rbase = wq * 32 + h * 16;           // the warp's first row = TMEM lane
    const int r0 = rbase + (lane >> 2), r1 = r0 + 8;
    const uint32_t lane_addr = uint32_t(rbase) << 16;
    const int cpair = 2 * (lane & 3);             // this thread's column pair in every 8 columns
    int2* rows_lh = reinterpret_cast<int2*>(smem + Dm::kOffRows);
    PairIter pi;
    pi.init(&p, w, &bars->ring, kClaimWarp, &wctx);
    int tA, tB, g, klo, khi;
    uint32_t s_cntA = 0, s_cntB = 0, o_cntA = 0, o_cntB = 0, st_cntA = 0, st_cntB = 0;
    bool ok = true;
    while (ok && pi.next(tA, tB, g, klo, khi)) {
      const int nx = tB >= 0 ? 2 : 1;
      const int n_kt = (khi - klo + BN - 1) / BN;
      Rows2 rsA, rsB;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        rsA.m_ref[k] = rsA.m_true[k] = rsB.m_ref[k] = rsB.m_true[k] = -INFINITY;
        rsA.l[k] = rsB.l[k] = 0.f;
      }
      // the allowed keys of this thread's rows in both tiles (none for a padding row),
      // kept in shared memory by the first thread of each row (read by the row's four)
      if ((lane & 3) == 0) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int t = x == 0 ? tA : tB;
          int4 tile = make_int4(0, 0, 0, 0);
          if (t >= 0) tile = p.tiles[t];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int rr = k == 0 ? r0 : r1;
            const int slot = rr / rows_per_slot;
            int2 lh = make_int2(0, 0);
            if (t >= 0 && slot < tile.y - tile.x) {
              const int4 ent = p.entries[tile.x + slot];
              lh = make_int2(ent.y, ent.z);
            }
            rows_lh[x * BM + rr] = lh;
          }
        }
      }
      __syncwarp();
      // key tile j of tile x: false when a wait gave up
      auto step = [&](Rows2& st, uint32_t& sc, const uint32_t oc, const int x, const int j) -> bool {
          const uint32_t tS = tmem + lane_addr + x * 128;
          const uint32_t tO = tmem + lane_addr + 256 + x * 128;   // O_X: rescaled in place on a new reference
          if (!warp_wait(&bars->s_ready[x], sc & 1, wctx, 1 * 10000 + __LINE__)) return false;
          ++sc;
          tc_fence_after();
          uint32_t v[64];
          tmem_ld16x256b_x16(tS, v);
          tmem_wait_ld();
          reg_fence<64>(v);
          // the rows' allowed columns in this key tile: [a, b); masked scores become -inf
          const int k0 = klo + j * BN;
          const int2 lh0 = rows_lh[x * BM + r0], lh1 = rows_lh[x * BM + r1];
          const int a0 = lh0.x - k0, b0 = lh0.y - k0, a1 = lh1.x - k0, b1 = lh1.y - k0;
          if (!__all_sync(0xffffffffu, a0 <= 0 && b0 >= BN && a1 <= 0 && b1 >= BN)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int col = 8 * i + cpair + e;
                v[4 * i + e] = (col >= a0 && col < b0) ? v[4 * i + e] : 0xff800000u;
                v[4 * i + 2 + e] = (col >= a1 && col < b1) ? v[4 * i + 2 + e] : 0xff800000u;
              }
            }
          }
          float mt0, mt1;
          row_max2(v, mt0, mt1);
          mt0 *= scale_log2;   // -inf: no allowed key of the row in this tile
          mt1 *= scale_log2;
          // a row's first allowed keys set its reference (its O and l are still zero);
          // a later maximum past the headroom rescales O and l to a new reference
          if (st.m_ref[0] == -INFINITY) st.m_ref[0] = mt0;
          if (st.m_ref[1] == -INFINITY) st.m_ref[1] = mt1;
          const bool over0 = mt0 > st.m_ref[0] + kHeadroomLog2, over1 = mt1 > st.m_ref[1] + kHeadroomLog2;
          if (__any_sync(0xffffffffu, over0 || over1)) {
            const float f0 = over0 ? fast_exp2(st.m_ref[0] - mt0) : 1.f;
            const float f1 = over1 ? fast_exp2(st.m_ref[1] - mt1) : 1.f;
            if (j > 0) {
              // the rows' O, after PV(j-1): 32 columns per 16x256b.x4 round trip
              if (!warp_wait(&bars->o_ready[x], (oc + j - 1) & 1, wctx, 1 * 10000 + __LINE__)) return false;
              tc_fence_after();
#pragma unroll 1
              for (int cch = 0; cch < D / 32; ++cch) {
                uint32_t o[16];
                tmem_ld16x256b_x4(tO + cch * 32, o);
                tmem_wait_ld();
                reg_fence<16>(o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  o[4 * i] = __float_as_uint(__uint_as_float(o[4 * i]) * f0);
                  o[4 * i + 1] = __float_as_uint(__uint_as_float(o[4 * i + 1]) * f0);
                  o[4 * i + 2] = __float_as_uint(__uint_as_float(o[4 * i + 2]) * f1);
                  o[4 * i + 3] = __float_as_uint(__uint_as_float(o[4 * i + 3]) * f1);
                }
                tmem_st16x256b_x4(tO + cch * 32, o);
              }
              tmem_wait_st();
            }
            st.l[0] *= f0;
            st.l[1] *= f1;
            if (over0) st.m_ref[0] = mt0;
            if (over1) st.m_ref[1] = mt1;
          }
          // P over the scores' first 64 columns (every score of these rows is in registers)
          exp_pack_store2(v, scale_log2, st.m_ref[0] == -INFINITY ? 0.f : -st.m_ref[0],
                          st.m_ref[1] == -INFINITY ? 0.f : -st.m_ref[1], tS, st.l[0], st.l[1]);
          st.m_true[0] = fmaxf(st.m_true[0], mt0);
          st.m_true[1] = fmaxf(st.m_true[1], mt1);
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&bars->p_ready[x]);
          return true;
      };
      for (int j = 0; j < n_kt && ok; ++j) {
#pragma unroll 1
        for (int x = 0; x < nx && ok; ++x) {
          Rows2 st = x == 0 ? rsA : rsB;
          uint32_t sc = x == 0 ? s_cntA : s_cntB;
          ok = step(st, sc, x == 0 ? o_cntA : o_cntB, x, j);
          if (x == 0) {
            rsA = st;
            s_cntA = sc;
          } else {
            rsB = st;
            s_cntB = sc;
          }
          if (ok && j == n_kt - 1) {
            // the tile's last key tile: its rows' statistics go to the epilogue warps at
            // once (the sum over the row's four threads, the true maximum, the reference)
            uint32_t stc = x == 0 ? st_cntA : st_cntB;
            float4* st4 = reinterpret_cast<float4*>(smem + Dm::kOffStats) + ((stc & 1) * 2 + x) * BM;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              float lk = st.l[k];
              lk += __shfl_xor_sync(0xffffffffu, lk, 1);
              lk += __shfl_xor_sync(0xffffffffu, lk, 2);
              if ((lane & 3) == 0) st4[k == 0 ? r0 : r1] = make_float4(lk, st.m_true[k], st.m_ref[k], 0.f);
            }
            __threadfence_block();
            warp_arrive(&bars->stats_ready[x][stc & 1]);
            if (x == 0) ++st_cntA; else ++st_cntB;
          }
        }
      }
      if (!ok) break;
      o_cntA += n_kt;
      if (nx == 2) o_cntB += n_kt;
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= 12) {
    // ------------------------------------------------------------ record epilogue
    // O_x of a finished tile from tensor memory to the record (times 1 / l), then the
    // record's m_c and l_c; the output columns are released to the MMA right after the
    // last TMEM read, so the next pair's first PV does not wait for the stores.
    const int wq = warp & 3;
    const int r = (wq << 5) + lane;   // row of the tile = TMEM lane
    const uint32_t lane_addr = uint32_t(wq << 5) << 16;
    float* scratch = reinterpret_cast<float*>(smem + Dm::kOffScratch) + wq * 1024;
    PairIter pi;
    pi.init(&p, w, &bars->ring, kClaimWarp, &wctx);
    int tA, tB, g, klo, khi;
    uint32_t pc[2] = {0, 0};
    bool ok = true;
    while (ok && pi.next(tA, tB, g, klo, khi)) {
      for (int x = 0; x < 2; ++x) {
        const int t = x == 0 ? tA : tB;
        if (t < 0) continue;
        const uint32_t tO = tmem + lane_addr + 256 + x * 128;
        const int4 tile = p.tiles[t];
        const int slot = r / rows_per_slot;
        const int within = r - slot * rows_per_slot;
        const int tt = within / p.G, hh = within - tt * p.G;
        const bool valid = slot < tile.y - tile.x;
        const int rec = valid ? ((tile.x + slot) * p.bs + tt) * p.Hq + g * p.G + hh : 0;
        if (!warp_wait(&bars->o_full[x], pc[x] & 1, wctx, 1 * 10000 + __LINE__)) { ok = false; break; }
        tc_fence_after();
        // O in rounds of two 32-column chunks (two rounds at D = 128, one at D = 64); the
        // output columns are released after the last round's TMEM reads, before its stores
        uint32_t va[32], vb[32];
        tmem_ld32(tO, va);
        tmem_ld32(tO + 32, vb);
        tmem_wait_ld();
        reg_fence<32>(va);
        reg_fence<32>(vb);
        if (D == 64) {
          tc_fence_before();
          warp_arrive(&bars->o_free[x]);
        }
        if (!warp_wait(&bars->stats_ready[x][pc[x] & 1], (pc[x] >> 1) & 1, wctx, 1 * 10000 + __LINE__)) {
          ok = false;
          break;
        }
        const float4 sx = reinterpret_cast<const float4*>(smem + Dm::kOffStats)[((pc[x] & 1) * 2 + x) * BM + r];
        ++pc[x];
        // 1 / l, and the record: m_c = the true maximum (natural units), l_c = the sum
        // relative to it (the halves' sums are relative to the common reference)
        const float l = sx.x + sx.w;
        const float4 st = make_float4(l > 0.f ? 1.f / l : 0.f, (l > 0.f) ? sx.y * kLn2 : -INFINITY,
                                      (l > 0.f) ? l * fast_exp2(sx.z - sx.y) : 0.f, 0.f);
        // stores of two 32-column chunks held in va, vb
        auto store2 = [&](int col) {
          if (p.partial_bf16) {
            if (valid) {
              lane_store32_bf16(static_cast<uint16_t*>(part_o) + size_t(rec) * D + col, va, st.x);
              lane_store32_bf16(static_cast<uint16_t*>(part_o) + size_t(rec) * D + col + 32, vb, st.x);
            }
            __syncwarp();   // valid differs across the warp's rows: converge before the next tcgen05.ld
          } else {
            float* dst = valid ? static_cast<float*>(part_o) + size_t(rec) * D + col : nullptr;
            warp_store_rows<32>(scratch, reinterpret_cast<const float*>(va), st.x, dst);
            warp_store_rows<32>(scratch, reinterpret_cast<const float*>(vb), st.x, valid ? dst + 32 : nullptr);
          }
        };
        store2(0);
        if (D == 128) {
          tmem_ld32(tO + 64, va);
          tmem_ld32(tO + 96, vb);
          tmem_wait_ld();
          reg_fence<32>(va);
          reg_fence<32>(vb);
          // every TMEM read of O_x done: the MMA may start the next pair's products into it
          tc_fence_before();
          warp_arrive(&bars->o_free[x]);
          store2(64);
        }
        if (valid) {
          part_m[rec] = st.y;
          part_l[rec] = st.z;
        }
      }
    }
    __syncwarp();
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
  if (tid == 0) p.timers[w * 2 + 1] = global_timer_ns();
}

}  // namespace

bool fwd_sm100_supported(const DevPlan& p) {
  const int rows = p.G * p.bs;
  return (p.d == 64 || p.d == 128) && rows % 8 == 0 && rows <= BM && tensor_maps_available();
}

namespace {

template <int D>
cudaError_t launch_fwd_sm100(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v, float scale,
                             void* part_o, float* part_m, float* part_l, cudaStream_t s) {
  constexpr uint32_t kSmem = Dims<D>::kSmemBytes;
  CUtensorMap tq, tk, tv;
  if (!make_bf16_map_3d(&tq, q, D, p.Hq, p.Nq, p.G, p.bs)) return cudaErrorInvalidValue;
  if (!make_bf16_map_3d(&tk, k, D, p.Hkv, p.N, 1, BN)) return cudaErrorInvalidValue;
  if (!make_bf16_map_3d(&tv, v, D, p.Hkv, p.N, 1, BN)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_partial_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmem));
  if (e != cudaSuccess) return e;
  // run-time claims start from item 0 at every launch
  if (p.dynamic && (e = cudaMemsetAsync(p.claim + 0, 0, sizeof(int), s)) != cudaSuccess) return e;
  fwd_partial_sm100_kernel<D><<<p.W, kThreads, kSmem, s>>>(tq, tk, tv, p, scale * kLog2e, part_o, part_m, part_l);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_partial_sm100(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     float scale, void* part_o, float* part_m, float* part_l, cudaStream_t s) {
  if (p.d == 64) return launch_fwd_sm100<64>(p, q, k, v, scale, part_o, part_m, part_l, s);
  return launch_fwd_sm100<128>(p, q, k, v, scale, part_o, part_m, part_l, s);
}

}  // namespace splitkv
