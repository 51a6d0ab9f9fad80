// Backward of the chunk partial attention on the 5th-generation tensor cores
// (tcgen05 / TMEM / TMA), head_dim 64 or 128.
//
// News page "Split-KV speeds diffusion drafter training by keeping long-context
// data local", section "Exchange the smaller side": keys and values stay local
// to their shard through the backward pass, and the query-side result is
// reduced across shards.  Here a shard is a KV chunk owned by one persistent CTA.
//
// Tensor memory (512 columns) cannot hold dK, dV, S, dP and dQ of a 128-key by
// 128-row tile pair at once, so the backward runs as two kernels that both
// recompute P = exp(s - lse) from the saved log-sum-exp:
//
//  dkdv kernel (KV-stationary, backward LPT schedule, whole chunks): for every
//    128-key tile of the chunk, for every query tile that meets it:
//      S^T = K Q^T, dP^T = V dO^T          (TMEM, keys as lanes; two commits)
//      P^T                                 (thread = key; bf16 over S^T, as soon
//                                           as S^T lands)
//      dV += P^T dO                        (A operand from TMEM, overlapping...)
//      dS^T = P^T (dP^T - Delta)           (... the dS^T pass; bf16 over dP^T)
//      dK += dS^T Q
//    then dK (times scale) and dV of the tile's keys go to global memory; keys
//    that no query reads get zeros.
//  dq kernel (Q-stationary, forward LPT schedule): for every query tile, over
//    the 128-key tiles of its chunk:
//      S = Q K^T (double-buffered), dP = dO V^T, dS = P (dP - Delta)
//      dQ += dS K                           (A operand from TMEM)
//    then scale * dQ is written once as the (chunk, block) entry's dq partial.
//
// Roles per CTA: warp 0 TMA producer, warp 1 MMA issuer (one thread), warp 2
// tensor-memory allocation, warp 3 prefetches the row metadata of upcoming query
// tiles into shared memory, warps 4-11 element-wise work in two warpgroups that
// split the 128 columns of every tile between them (thread = TMEM lane; warpgroup
// h takes columns 64h..64h+63).  Each warpgroup writes its bf16 results into its
// own columns (the MMA addresses the 16-wide K-steps one by one), so neither
// overwrites scores the other has not read yet.  The dK/dV kernel (384 threads)
// writes dK, dV from the element-wise warps after each key tile; the dQ kernel
// (512 threads) has warps 12-15 of its own for the dq-partial epilogue, so the
// element-wise warps go on with the next query tile meanwhile.  Waits are bounded;
// a timeout is recorded in the plan's status word and every role winds down.
#include <cfloat>
#include <cstring>

#include "sm100.cuh"
#include "splitkv.h"
#include "splitkv_internal.h"

namespace splitkv {
namespace {

using namespace sm100;

constexpr int BT = 128;                // keys per key tile = rows per query tile
constexpr int kThreads = 384;
constexpr uint32_t kHalf = 128 * 128;  // one 64-column half of a 128-row bf16 tile
constexpr uint32_t kIdescKM = idesc_bf16_f32(128, 128, 0);  // B K-major

// Sizes that follow the head dimension D (64 or 128): a 128-row bf16 tile of D
// columns is D / 64 halves of 16 KB; the products into dK, dV, dQ have N = D.
// Shared memory: 6 tiles | row metadata (8 KB) | epilogue scratch (8 x 2 KB: one
// per element-wise warp of the dK/dV kernel, one per epilogue warp of the dQ
// kernel) | barriers.
template <int D>
struct Dims {
  static_assert(D == 64 || D == 128, "head dimension");
  static constexpr uint32_t kTile = uint32_t(D / 64) * kHalf;
  static constexpr uint32_t kIdescMN = idesc_bf16_f32(128, D, 1);   // B MN-major, N = D
  static constexpr uint32_t kOffMeta = 6 * kTile;
  static constexpr uint32_t kOffScratch = kOffMeta + 8192;
  static constexpr uint32_t kOffBars = kOffScratch + 8 * 2048;
  static constexpr uint32_t kSmemBytes = kOffBars + 256 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};


// K-major SW128 descriptor of the k-th 16-column step of a 128-row tile.
__device__ __forceinline__ uint64_t kmajor(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
}
// MN-major SW128 descriptor of the k-th 16-row step of a 128-row tile (N = 128 columns).
__device__ __forceinline__ uint64_t mnmajor(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + kk * 2048, kHalf, 1024);
}
// TMEM column (relative to a 128-column score buffer) of the bf16 pairs of the
// k-th 16-wide K-step: steps 0..3 (written by warpgroup 0) sit in columns 0..31,
// steps 4..7 (warpgroup 1) in columns 64..95 -- inside each warpgroup's own
// half of the buffer, over scores it has already read.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk < 4 ? 0u : 64u) + 8u * uint32_t(kk & 3); }

// Row metadata of query-tile row r (rows ordered slot, token, head).
struct RowMeta {
  bool valid;
  int lo, hi, rec;
  size_t qrow;
};
__device__ __forceinline__ RowMeta row_meta(const DevPlan& p, const int4& tile, int g, int r) {
  RowMeta m;
  const int rps = p.G * p.bs;
  const int slot = r / rps;
  const int within = r - slot * rps;
  const int tt = within / p.G, hh = within - tt * p.G;
  m.valid = slot < tile.y - tile.x;
  m.lo = m.hi = m.rec = 0;
  m.qrow = 0;
  if (m.valid) {
    const int e = tile.x + slot;
    const int4 ent = p.entries[e];
    m.lo = ent.y;
    m.hi = ent.z;
    m.rec = (e * p.bs + tt) * p.Hq + g * p.G + hh;
    m.qrow = size_t(ent.x * p.bs + tt) * p.Hq + g * p.G + hh;
  }
  return m;
}

// TMA of one query tile's rows (Q or dO layout) into a 128-row SW128 tile
// (D / 64 halves).  Slots past the tile's last block are loaded from token
// coordinate Nq, outside the tensor, so that the hardware fills them with
// zeros: the dK/dV products contract over all 128 rows.
template <int D>
__device__ __forceinline__ void load_query_tile(const DevPlan& p, const int4& tile, int g, uint8_t* dst,
                                                const CUtensorMap* map, uint64_t* bar) {
  const int rps = p.G * p.bs;
  const uint32_t slot_bytes = uint32_t(rps) * 128;
  const int n = tile.y - tile.x;
  for (int s = 0; s < BT / rps; ++s) {
    const int z = s < n ? p.entries[tile.x + s].x * p.bs : p.Nq;
    for (int dh = 0; dh < D / 64; ++dh)
      tma_load_3d(dst + dh * kHalf + s * slot_bytes, map, bar, dh * 64, g * p.G, z);
  }
}

__device__ __forceinline__ void setup_common(uint64_t* bars, int nbars, const uint32_t* counts, uint32_t* tmem_slot,
                                             int warp) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < nbars; ++i) mbar_init(&bars[i], counts[i]);
    mbar_fence_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// The dQ pass takes one exponential pair in eight on the FMA-pipe polynomial (measured:
// 1/8 and all-MUFU ~2 % faster than the dK/dV pass's one in four, one in two 5 % slower).
constexpr int kPolyEveryDq = 8;

// dq kernel, half hf of one key tile for one row (thread = TMEM lane): dS =
// P (dP - Delta) with P = exp2(s * c - lse2), zero outside the row's columns
// [a, b) of the tile; bf16 pairs of dS go to packed_col() of the score buffer.
template <bool kMasked>
__device__ __forceinline__ void ds_tile(uint32_t tS, uint32_t tdP, int hf, int a, int b, float c, float l2,
                                        float dl) {
#pragma unroll 1
  for (int q = 2 * hf; q < 2 * hf + 2; ++q) {   // 32 keys per TMEM round trip
    uint32_t sv[32], dpv[32];
    tmem_ld32(tS + q * 32, sv);
    tmem_ld32(tdP + q * 32, dpv);
    tmem_wait_ld();
    reg_fence<32>(sv);
    reg_fence<32>(dpv);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int col = q * 32 + 2 * i;
      float x0, x1, d0, d1, g0, g1;
      ffma2(x0, x1, __uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]), c, c, -l2, -l2);
      float p0, p1;
      exp2_pair((i % kPolyEveryDq) == 1, x0, x1, p0, p1);
      if (kMasked) {
        p0 = (col >= a && col < b) ? p0 : 0.f;
        p1 = (col + 1 >= a && col + 1 < b) ? p1 : 0.f;
      }
      fadd2(d0, d1, __uint_as_float(dpv[2 * i]), __uint_as_float(dpv[2 * i + 1]), -dl, -dl);
      fmul2(g0, g1, p0, p1, d0, d1);
      pk[i] = pack_bf16(g0, g1);
    }
    tmem_st16p(tS + packed_col(2 * q), pk);
  }
}

// dkdv kernel, rows 64hf..64hf+63 of one query tile for one key (thread = TMEM
// lane), first half of the element-wise step: P^T = exp2(s * c - lse2[row]),
// zero for rows whose slot bit (slot = row >> lg) is clear.  P stays in pv
// (fp32, for dS^T) and goes as bf16 pairs to packed_col() of S^T.  The rows
// are the columns of S^T, so every element needs its own row statistic: the
// 32 of a TMEM round trip are loaded together (eight 16-byte shared loads)
// before the scores, not one per element inside the loop.
template <bool kMasked>
__device__ __forceinline__ void pt_tile(uint32_t tSt, int hf, uint32_t smask, int lg, const float* l2tile, float c,
                                        float (&pv)[64]) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {   // 32 rows per TMEM round trip
    const int q = 2 * hf + qq;
    float l2[32];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 v = reinterpret_cast<const float4*>(l2tile + q * 32)[k];
      l2[4 * k] = v.x;
      l2[4 * k + 1] = v.y;
      l2[4 * k + 2] = v.z;
      l2[4 * k + 3] = v.w;
    }
    uint32_t sv[32];
    tmem_ld32(tSt + q * 32, sv);
    tmem_wait_ld();
    reg_fence<32>(sv);
    reg_fence<32>(reinterpret_cast<uint32_t*>(l2));
    uint32_t pp[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int row = q * 32 + 2 * i;
      float x0, x1;
      ffma2(x0, x1, __uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]), c, c, -l2[2 * i], -l2[2 * i + 1]);
      float p0, p1;
      exp2_pair((i % kPolyEvery) == 1, x0, x1, p0, p1);
      if (kMasked) {
        const bool in = (smask >> (row >> lg)) & 1u;
        p0 = in ? p0 : 0.f;
        p1 = in ? p1 : 0.f;
      }
      pv[qq * 32 + 2 * i] = p0;
      pv[qq * 32 + 2 * i + 1] = p1;
      pp[i] = pack_bf16(p0, p1);
    }
    tmem_st16p(tSt + packed_col(2 * q), pp);
  }
}

// Second half: dS^T = P^T (dP^T - Delta[row]) as bf16 pairs to packed_col() of dP^T.
__device__ __forceinline__ void dst_tile(uint32_t tdPt, int hf, const float* dltile, const float (&pv)[64]) {
#pragma unroll
  for (int qq = 0; qq < 2; ++qq) {
    const int q = 2 * hf + qq;
    float dl[32];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 v = reinterpret_cast<const float4*>(dltile + q * 32)[k];
      dl[4 * k] = v.x;
      dl[4 * k + 1] = v.y;
      dl[4 * k + 2] = v.z;
      dl[4 * k + 3] = v.w;
    }
    uint32_t dpv[32];
    tmem_ld32(tdPt + q * 32, dpv);
    tmem_wait_ld();
    reg_fence<32>(dpv);
    reg_fence<32>(reinterpret_cast<uint32_t*>(dl));
    uint32_t pd[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float d0, d1, g0, g1;
      fadd2(d0, d1, __uint_as_float(dpv[2 * i]), __uint_as_float(dpv[2 * i + 1]), -dl[2 * i], -dl[2 * i + 1]);
      fmul2(g0, g1, pv[qq * 32 + 2 * i], pv[qq * 32 + 2 * i + 1], d0, d1);
      pd[i] = pack_bf16(g0, g1);
    }
    tmem_st16p(tdPt + packed_col(2 * q), pd);
  }
}

// ============================================================================
// dkdv kernel
// ============================================================================
struct DkdvBars {
  uint64_t kv_full, kv_empty, qd_full[2], qd_empty[2], st_ready, dpt_ready, pt_ready, dst_ready, dkv_ready,
      dkv_free, mma_done, meta_ready[2], meta_free[2];
  ClaimRing ring;   // run-time claims: producer -> MMA thread, metadata warp, 8 element-wise warps
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int kDkdvNumBars = 17;
static_assert(sizeof(DkdvBars) <= 256, "barrier block");
// consumers of the claim ring in both backward kernels: the MMA thread, warp 3, warps 4-11
constexpr uint32_t kClaimConsumers = 1 + 1 + 8;

// The item sequence of one role of the dK/dV kernel: the worker's items of the
// backward schedule, or its run-time claims.
__device__ __forceinline__ void bwd_item_seq(ItemSeq& s, const DevPlan& p, int w, ClaimRing* ring, int role) {
  if (p.dynamic)
    s.init_claims(ring, p.claim + 1, p.n_bwd_items, role);
  else
    s.init_static(p.bwd_worker_ptr[w], p.bwd_worker_ptr[w + 1]);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                          DevPlan p, const float* __restrict__ lse, const float* __restrict__ delta, float scale,
                          float* __restrict__ dk, float* __restrict__ dv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using Dm = Dims<D>;
  constexpr uint32_t kTile = Dm::kTile;
  constexpr uint32_t kIdescMN = Dm::kIdescMN;
  uint8_t* sK = smem;
  uint8_t* sV = smem + kTile;
  uint8_t* sQ = smem + 2 * kTile;   // [2 stages]
  uint8_t* sdO = smem + 4 * kTile;  // [2 stages]
  float* meta_l2 = reinterpret_cast<float*>(smem + Dm::kOffMeta);               // [2][128] lse2 per row
  float* meta_dl = reinterpret_cast<float*>(smem + Dm::kOffMeta + 1024);        // [2][128] delta per row
  int2* meta_slot = reinterpret_cast<int2*>(smem + Dm::kOffMeta + 2048);         // [2][16] (lo, hi) per slot
  DkdvBars* B = reinterpret_cast<DkdvBars*>(smem + Dm::kOffBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int w = blockIdx.x;
  volatile int* abort_flag = &B->abort_flag;
  const WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};
  if (tid == 0) {
    p.timers[(p.W + w) * 2 + 0] = global_timer_ns();
    B->abort_flag = 0;
  }
  {
    // commits count 1; element-wise / metadata signals count warps (warp_arrive)
    const uint32_t counts[kDkdvNumBars] = {1, 1, 1, 1, 1, 1, 1, 1, 8, 8, 1, 8, 1, 1, 1, 8, 8};
    if (tid == 0) claim_ring_init(&B->ring, kClaimConsumers);
    setup_common(&B->kv_full, kDkdvNumBars, counts, &B->tmem_base, warp);
  }
  const uint32_t tmem = B->tmem_base;
  const size_t kv_row = size_t(p.Hkv) * D;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t kt_count = 0, qd_count = 0;
      bool ok = true;
      ItemSeq seq;
      bwd_item_seq(seq, p, w, &B->ring, kClaimProducer);
      int idx;
      while (ok && seq.next(idx, wctx, 2 * 10000 + __LINE__)) {
        const int4 item = p.bwd_items[idx];
        const int g = item.y, c0 = item.x * p.C, c1 = min(c0 + p.C, p.N);
        for (int k0 = c0; ok && k0 < c1; k0 += BT) {
          if (!mbar_wait(&B->kv_empty, (kt_count & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          mbar_expect_tx(&B->kv_full, 2 * kTile);
          for (int dh = 0; dh < D / 64; ++dh) {
            tma_load_3d(sK + dh * kHalf, &tm_k, &B->kv_full, dh * 64, g, k0);
            tma_load_3d(sV + dh * kHalf, &tm_v, &B->kv_full, dh * 64, g, k0);
          }
          ++kt_count;
          for (int t = item.z; t < item.w; ++t) {
            const int4 tile = p.tiles[t];
            if (!(tile.z < k0 + BT && tile.w > k0)) continue;
            const int s = qd_count & 1;
            if (!mbar_wait(&B->qd_empty[s], ((qd_count >> 1) & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
            mbar_expect_tx(&B->qd_full[s], 2 * kTile);
            load_query_tile<D>(p, tile, g, sQ + s * kTile, &tm_q, &B->qd_full[s]);
            load_query_tile<D>(p, tile, g, sdO + s * kTile, &tm_do, &B->qd_full[s]);
            ++qd_count;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      if (kt_count > 0) mbar_drain(&B->kv_full, (kt_count - 1) & 1, wctx, 2 * 10000 + __LINE__);
      for (uint32_t c = qd_count >= 2 ? qd_count - 2 : 0; c < qd_count; ++c) mbar_drain(&B->qd_full[c & 1], (c >> 1) & 1, wctx, 2 * 10000 + __LINE__);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), adO = smem_u32(sdO);
      uint32_t kt_count = 0, qd_count = 0, pds_cnt = 0, dkvf_cnt = 0;
      bool ok = true;
      ItemSeq seq;
      bwd_item_seq(seq, p, w, &B->ring, kClaimThread);
      int idx;
      while (ok && seq.next(idx, wctx, 2 * 10000 + __LINE__)) {
        const int4 item = p.bwd_items[idx];
        const int c0 = item.x * p.C, c1 = min(c0 + p.C, p.N);
        for (int k0 = c0; ok && k0 < c1; k0 += BT) {
          if (!mbar_wait(&B->kv_full, kt_count & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          tc_fence_after();
          int u = 0;
          bool s_issued = false;   // S^T of this pair was issued ahead, right after the previous dV
          for (int t = item.z; t < item.w; ++t) {
            const int4 tile = p.tiles[t];
            if (!(tile.z < k0 + BT && tile.w > k0)) continue;
            const int s = qd_count & 1;
            if (!s_issued) {
              if (!mbar_wait(&B->qd_full[s], (qd_count >> 1) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
              tc_fence_after();
              // S^T = K Q^T (cols 0..127); the P^T pass starts when it lands
              for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + 0, kmajor(aK, kk), kmajor(aQ + s * kTile, kk), kIdescKM, kk > 0 ? 1u : 0u);
              mma_commit(&B->st_ready);
            }
            s_issued = false;
            // dP^T = V dO^T (cols 128..255): after dK of the previous pair, which read dS^T there
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + 128, kmajor(aV, kk), kmajor(adO + s * kTile, kk), kIdescKM, kk > 0 ? 1u : 0u);
            mma_commit(&B->dpt_ready);
            // the next pair of this key tile, if any
            int tn = -1;
            for (int t2 = t + 1; t2 < item.w; ++t2) {
              const int4 tl2 = p.tiles[t2];
              if (tl2.z < k0 + BT && tl2.w > k0) {
                tn = t2;
                break;
              }
            }
            // K and V are read only by S^T / dP^T: release them after the key tile's last pair
            if (tn < 0) mma_commit(&B->kv_empty);
            if (!mbar_wait(&B->pt_ready, pds_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
            if (u == 0) {
              if (!mbar_wait(&B->dkv_free, (dkvf_cnt & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
              ++dkvf_cnt;
            }
            tc_fence_after();
            // dV (cols 384..) += P^T dO while dS^T is formed -- A operand from TMEM
            for (int kk = 0; kk < BT / 16; ++kk)
              mma_ts(tmem + 384, tmem + 0 + packed_col(kk), mnmajor(adO + s * kTile, kk), kIdescMN,
                     (u > 0 || kk > 0) ? 1u : 0u);
            if (tn >= 0) {
              // the next pair's S^T right behind dV, which is the last reader of this pair's
              // P^T in cols 0..127 (the dS^T pass keeps P in registers): its P^T pass can then
              // start as soon as the element-wise warps finish this pair, while dK runs
              const int s1 = (qd_count + 1) & 1;
              if (!mbar_wait(&B->qd_full[s1], ((qd_count + 1) >> 1) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
              tc_fence_after();
              for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + 0, kmajor(aK, kk), kmajor(aQ + s1 * kTile, kk), kIdescKM, kk > 0 ? 1u : 0u);
              mma_commit(&B->st_ready);
              s_issued = true;
            }
            if (!mbar_wait(&B->dst_ready, pds_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
            ++pds_cnt;
            tc_fence_after();
            // dK (cols 256..) += dS^T Q
            for (int kk = 0; kk < BT / 16; ++kk)
              mma_ts(tmem + 256, tmem + 128 + packed_col(kk), mnmajor(aQ + s * kTile, kk), kIdescMN,
                     (u > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&B->qd_empty[s]);
            ++qd_count;
            ++u;
          }
          if (!ok) break;
          if (u > 0) mma_commit(&B->dkv_ready);
          else mma_commit(&B->kv_empty);   // no pair met this key tile
          ++kt_count;
        }
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&B->mma_done);
      mbar_drain(&B->mma_done, 0, wctx, 2 * 10000 + __LINE__);
    }
  } else if (warp == 3) {
    // metadata of the query tiles, in the element-wise order, up to two tiles ahead
    uint32_t mcount = 0;
    bool ok = true;
    ItemSeq seq;
    bwd_item_seq(seq, p, w, &B->ring, kClaimWarp);
    int idx;
    while (ok && seq.next(idx, wctx, 2 * 10000 + __LINE__)) {
      const int4 item = p.bwd_items[idx];
      const int g = item.y, c0 = item.x * p.C, c1 = min(c0 + p.C, p.N);
      for (int k0 = c0; ok && k0 < c1; k0 += BT) {
        for (int t = item.z; t < item.w; ++t) {
          const int4 tile = p.tiles[t];
          if (!(tile.z < k0 + BT && tile.w > k0)) continue;
          const int s = mcount & 1;
          if (!warp_wait(&B->meta_free[s], ((mcount >> 1) & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          const int rps = p.G * p.bs;
          for (int rr = lane; rr < BT; rr += 32) {
            const RowMeta m = row_meta(p, tile, g, rr);
            float l2 = INFINITY, dl = 0.f;
            if (m.valid) {
              const float L = lse[m.qrow];
              l2 = (L == -INFINITY) ? INFINITY : L * kLog2e;
              dl = delta[m.qrow];
            }
            meta_l2[s * 128 + rr] = l2;
            meta_dl[s * 128 + rr] = dl;
            if (rr % rps == 0) meta_slot[s * 16 + rr / rps] = make_int2(m.lo, m.hi);
          }
          warp_arrive(&B->meta_ready[s]);
          ++mcount;
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= 4) {
    const int hf = (warp - 4) >> 2;           // warpgroup: rows 64hf..64hf+63 of every query tile
    const int r = ((warp & 3) << 5) + lane;   // key of the tile = TMEM lane
    const uint32_t lane_addr = uint32_t((warp & 3) << 5) << 16;
    const uint32_t tSt = tmem + lane_addr;          // S^T / P^T
    const uint32_t tdPt = tmem + lane_addr + 128;   // dP^T / dS^T
    const uint32_t tAcc = tmem + lane_addr + 256 + hf * 128;   // dK (warpgroup 0) or dV (warpgroup 1)
    const float scale_log2 = scale * kLog2e;
    // chunks no block reads: zeros for every KV head
    const int et = tid - 128;
    for (int z = w; z < p.num_zero_chunks; z += p.Wb) {
      const int c = p.zero_chunks[z];
      const size_t first = size_t(c) * p.C * kv_row;
      const size_t last = size_t(min(c * p.C + p.C, p.N)) * kv_row;
      for (size_t i = first + size_t(et) * 4; i < last; i += size_t(256) * 4) {
        *reinterpret_cast<float4*>(dk + i) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(dv + i) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    uint32_t qd_count = 0, st_cnt = 0, dkv_cnt = 0;
    bool ok = true;
    ItemSeq seq;
    bwd_item_seq(seq, p, w, &B->ring, kClaimWarp);
    int idx;
    while (ok && seq.next(idx, wctx, 2 * 10000 + __LINE__)) {
      const int4 item = p.bwd_items[idx];
      const int g = item.y, c0 = item.x * p.C, c1 = min(c0 + p.C, p.N);
      for (int k0 = c0; ok && k0 < c1; k0 += BT) {
        const int key = k0 + r;
        int n_meet = 0;
        for (int t = item.z; t < item.w; ++t) {
          const int4 tile = p.tiles[t];
          if (!(tile.z < k0 + BT && tile.w > k0)) continue;
          const int s = qd_count & 1;
          const int rps = p.G * p.bs;
          // the tile's row metadata, prefetched by warp 3
          if (!warp_wait(&B->meta_ready[s], (qd_count >> 1) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          // slots (blocks) that may read this thread's key: one bit per slot.  Padding
          // slots count as "in": their rows have lse2 = +inf, so P = 0 there anyway.
          const int nslots = BT / rps;             // rps is a power of two (8 .. 128)
          const int lg = 31 - __clz(rps);
          uint32_t smask = ~((1u << (tile.y - tile.x)) - 1u);
          for (int sl = 0; sl < tile.y - tile.x; ++sl) {
            const int2 lh = meta_slot[s * 16 + sl];
            if (key >= lh.x && key < lh.y) smask |= 1u << sl;
          }
          const uint32_t all = nslots >= 32 ? 0xffffffffu : ((1u << nslots) - 1u);
          // warp-uniform choice: both paths issue warp-collective tcgen05.ld/st
          const bool all_in = __all_sync(0xffffffffu, (smask & all) == all);
          if (!warp_wait(&B->st_ready, st_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          tc_fence_after();
          float pv[64];
          if (all_in)
            pt_tile<false>(tSt, hf, smask, lg, meta_l2 + s * 128, scale_log2, pv);
          else
            pt_tile<true>(tSt, hf, smask, lg, meta_l2 + s * 128, scale_log2, pv);
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&B->pt_ready);
          if (!warp_wait(&B->dpt_ready, st_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          ++st_cnt;
          tc_fence_after();
          dst_tile(tdPt, hf, meta_dl + s * 128, pv);
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&B->dst_ready);
          warp_arrive(&B->meta_free[s]);
          ++qd_count;
          ++n_meet;
        }
        if (!ok) break;
        // epilogue of the key tile: warpgroup 0 writes dK * scale, warpgroup 1 dV
        // (zeros when no query met the tile)
        float* dst = (hf == 0 ? dk : dv) + (size_t(key) * p.Hkv + g) * D;
        const float f = hf == 0 ? scale : 1.f;
        const bool own = key < c1;
        if (n_meet > 0) {
          if (!warp_wait(&B->dkv_ready, dkv_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          ++dkv_cnt;
          tc_fence_after();
          float* scratch = reinterpret_cast<float*>(smem + Dm::kOffScratch) + (warp - 4) * 512;
          if (__all_sync(0xffffffffu, own)) {
            // the warp's 32 keys all belong to this chunk (and lie below N): bulk
            // tensor stores of 32 keys x 16 columns
            const CUtensorMap* map = hf == 0 ? &tm_dk : &tm_dv;
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
              uint32_t a[16];
              tmem_ld16(tAcc + cc * 16, a);
              tmem_wait_ld();
              reg_fence<16>(a);
              warp_bulk_store16<0>(scratch, a, f, map, cc * 16, g, k0 + ((warp & 3) << 5));
            }
          } else {
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
              uint32_t a[16];
              tmem_ld16(tAcc + cc * 16, a);
              tmem_wait_ld();
              reg_fence<16>(a);
              warp_store_rows<16>(scratch, reinterpret_cast<const float*>(a), f, own ? dst + cc * 16 : nullptr);
            }
          }
          tc_fence_before();
          warp_arrive(&B->dkv_free);
        } else if (own) {
          for (int i = 0; i < D; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    // bulk stores of this warp complete before the CTA exits
    if (lane == 0) bulk_wait0();
    __syncwarp();
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
  if (tid == 0) p.timers[(p.W + w) * 2 + 1] = global_timer_ns();
}

// ============================================================================
// dq kernel
// ============================================================================
// K goes through a ring of three stages (read by S and by dQ += dS K, so a stage frees
// late), V through one (read by dP only); the stages' shared memory equals two of each.
constexpr int kDqKStages = 3;
struct DqBars {
  uint64_t qd_full, qd_empty, k_full[kDqKStages], v_full, k_empty[kDqKStages], v_empty, s_ready[2], dp_ready,
      ds_ready, dq_ready, dq_free, mma_done, meta_ready[2], meta_free[2];
  ClaimRing ring;   // run-time claims: producer -> MMA thread, metadata warp, 8 element-wise warps
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int kDqNumBars = 21;
// dQ kernel roles (512 threads): warps 0-3 as in the dK/dV kernel, 4-11 element-wise,
// 12-15 the dq-partial epilogue; claim-ring consumers: MMA thread, warp 3, warps 4-15
constexpr int kDqThreads = 512;
constexpr uint32_t kDqClaimConsumers = 1 + 1 + 8 + 4;
static_assert(sizeof(DqBars) <= 256, "barrier block");

// Per-row metadata of a query tile for the dq kernel (shared memory).
struct DqRow {
  int lo, hi, rec, valid;
  float l2, dl;
};

// The query tiles of a worker's forward schedule (or of the forward items it
// claims at run time), one at a time.
struct TileIter {
  const DevPlan* p;
  const WaitCtx* wc;
  ItemSeq seq;
  int t, t_end, g;
  __device__ void init(const DevPlan* plan, int w, ClaimRing* ring, int role, const WaitCtx* wctx) {
    p = plan;
    wc = wctx;
    if (plan->dynamic)
      seq.init_claims(ring, plan->claim + 2, plan->n_fwd_items, role);
    else
      seq.init_static(plan->fwd_worker_ptr[w], plan->fwd_worker_ptr[w + 1]);
    t = t_end = 0;
    g = 0;
  }
  // false at the end (or when a claim wait gave up, which the wait recorded)
  __device__ bool next(int& tile_id, int& head) {
    while (t >= t_end) {
      int idx;
      if (!seq.next(idx, *wc, 2 * 10000 + __LINE__)) return false;
      const int4 item = p->fwd_items[idx];
      g = item.y;
      t = item.z;
      t_end = item.w;
    }
    tile_id = t++;
    head = g;
    return true;
  }
};

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_dq, DevPlan p, const float* __restrict__ lse,
                        const float* __restrict__ delta, float scale, int bulk, void* __restrict__ dq_part) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using Dm = Dims<D>;
  constexpr uint32_t kTile = Dm::kTile;
  constexpr uint32_t kIdescMN = Dm::kIdescMN;
  uint8_t* sQ = smem;
  uint8_t* sdO = smem + kTile;
  uint8_t* sK = smem + 2 * kTile;   // [kDqKStages stages]
  uint8_t* sV = smem + (2 + kDqKStages) * kTile;
  DqRow* meta = reinterpret_cast<DqRow*>(smem + Dm::kOffMeta);   // [2][128]
  DqBars* B = reinterpret_cast<DqBars*>(smem + Dm::kOffBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int w = blockIdx.x;
  volatile int* abort_flag = &B->abort_flag;
  const WaitCtx wctx{abort_flag, p.status, p.wait_limit_ns};
  if (tid == 0) {
    p.timers[(p.W + p.Wb + w) * 2 + 0] = global_timer_ns();
    B->abort_flag = 0;
  }
  {
    // commits count 1; element-wise / metadata signals count warps (warp_arrive)
    const uint32_t counts[kDqNumBars] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 8, 1, 4, 1, 1, 1, 8, 8};
    if (tid == 0) claim_ring_init(&B->ring, kDqClaimConsumers);
    setup_common(&B->qd_full, kDqNumBars, counts, &B->tmem_base, warp);
  }
  const uint32_t tmem = B->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      TileIter ti;
      ti.init(&p, w, &B->ring, kClaimProducer, &wctx);
      int t, g;
      uint32_t tile_count = 0, kv_count = 0, q_issued = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      // key tile c of this CTA, in the order the MMA thread reads them: K (its stage of
      // three frees after dQ += dS K of key tile c - 3), then V (its one stage frees once
      // dP of key tile c - 1 has read it)
      auto load_kv = [&](uint32_t c, int k0) -> bool {
        const int s = int(c % kDqKStages);
        if (!mbar_wait(&B->k_empty[s], ((c / kDqKStages) & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) return false;
        mbar_expect_tx(&B->k_full[s], kTile);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_3d(sK + s * kTile + dh * kHalf, &tm_k, &B->k_full[s], dh * 64, g, k0);
        ++k_issued;
        if (!mbar_wait(&B->v_empty, (c & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) return false;
        mbar_expect_tx(&B->v_full, kTile);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_3d(sV + dh * kHalf, &tm_v, &B->v_full, dh * 64, g, k0);
        ++v_issued;
        return true;
      };
      while (ok && ti.next(t, g)) {
        const int4 tile = p.tiles[t];
        const int n_kt = (tile.w - tile.z + BT - 1) / BT;
        // the tile's first key tile needs only free stages: request it before the Q / dO
        // buffer frees (the previous tile's last S and dP), so that it lands meanwhile
        if (!load_kv(kv_count, tile.z)) { ok = false; break; }
        if (!mbar_wait(&B->qd_empty, (tile_count & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
        mbar_expect_tx(&B->qd_full, 2 * kTile);
        load_query_tile<D>(p, tile, g, sQ, &tm_q, &B->qd_full);
        load_query_tile<D>(p, tile, g, sdO, &tm_do, &B->qd_full);
        ++q_issued;
        for (int j = 1; j < n_kt && ok; ++j)
          if (!load_kv(kv_count + j, tile.z + j * BT)) ok = false;
        if (!ok) break;
        kv_count += n_kt;
        ++tile_count;
      }
      if (!ok) *abort_flag = 1;
      if (q_issued > 0) mbar_drain(&B->qd_full, (q_issued - 1) & 1, wctx, 2 * 10000 + __LINE__);
      for (uint32_t c = k_issued >= kDqKStages ? k_issued - kDqKStages : 0; c < k_issued; ++c)
        mbar_drain(&B->k_full[c % kDqKStages], (c / kDqKStages) & 1, wctx, 2 * 10000 + __LINE__);
      if (v_issued > 0) mbar_drain(&B->v_full, (v_issued - 1) & 1, wctx, 2 * 10000 + __LINE__);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), adO = smem_u32(sdO);
      TileIter ti;
      ti.init(&p, w, &B->ring, kClaimThread, &wctx);
      int t, g;
      uint32_t tile_count = 0, kv_count = 0, ds_cnt = 0, dqf_cnt = 0;
      bool ok = true;
      while (ok && ti.next(t, g)) {
        const int4 tile = p.tiles[t];
        const int n_kt = (tile.w - tile.z + BT - 1) / BT;
        if (!mbar_wait(&B->qd_full, tile_count & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
        const uint32_t c0 = kv_count;
        {
          const int s = c0 & 1, ks = int(c0 % kDqKStages);   // S buffer, K stage
          if (!mbar_wait(&B->k_full[ks], (c0 / kDqKStages) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          tc_fence_after();
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + s * 128, kmajor(aQ, kk), kmajor(aK + ks * kTile, kk), kIdescKM, kk > 0 ? 1u : 0u);
          mma_commit(&B->s_ready[s]);
          if (!mbar_wait(&B->v_full, c0 & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          tc_fence_after();
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + 256, kmajor(adO, kk), kmajor(aV, kk), kIdescKM, kk > 0 ? 1u : 0u);
          mma_commit(&B->dp_ready);
          mma_commit(&B->v_empty);   // V is read by dP only
        }
        for (int j = 0; j < n_kt; ++j) {
          const uint32_t c = c0 + j;
          const int s = c & 1, s1 = (c + 1) & 1;   // S buffers
          const int ks = int(c % kDqKStages), ks1 = int((c + 1) % kDqKStages);   // K stages
          const bool more = j + 1 < n_kt;
          if (more) {   // next S into the other buffer while this tile's dS is formed
            if (!mbar_wait(&B->k_full[ks1], ((c + 1) / kDqKStages) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
            tc_fence_after();
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + s1 * 128, kmajor(aQ, kk), kmajor(aK + ks1 * kTile, kk), kIdescKM, kk > 0 ? 1u : 0u);
            mma_commit(&B->s_ready[s1]);
          }
          if (!mbar_wait(&B->ds_ready, ds_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
          ++ds_cnt;
          // the next dP first (the element-wise warps have read this one's dP): their next
          // pass then waits for one product, not two; dQ += dS K runs during that pass
          if (more) {
            if (!mbar_wait(&B->v_full, (c + 1) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
            tc_fence_after();
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + 256, kmajor(adO, kk), kmajor(aV, kk), kIdescKM, kk > 0 ? 1u : 0u);
            mma_commit(&B->dp_ready);
            mma_commit(&B->v_empty);
            if (j + 2 == n_kt) mma_commit(&B->qd_empty);   // Q, dO: no further reader after this S / dP
          }
          if (j == 0) {
            if (!mbar_wait(&B->dq_free, (dqf_cnt & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
            ++dqf_cnt;
          }
          tc_fence_after();
          // dQ (cols 384..) += dS K -- dS in TMEM (columns 0..63 of S buffer s), K MN-major
          for (int kk = 0; kk < BT / 16; ++kk)
            mma_ts(tmem + 384, tmem + s * 128 + packed_col(kk), mnmajor(aK + ks * kTile, kk), kIdescMN,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B->k_empty[ks]);   // K is read by S and by dQ += dS K
        }
        if (!ok) break;
        mma_commit(&B->dq_ready);
        if (n_kt == 1) mma_commit(&B->qd_empty);
        kv_count += n_kt;
        ++tile_count;
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&B->mma_done);
      mbar_drain(&B->mma_done, 0, wctx, 2 * 10000 + __LINE__);
    }
  } else if (warp == 3) {
    // row metadata of upcoming query tiles, up to two tiles ahead
    TileIter ti;
    ti.init(&p, w, &B->ring, kClaimWarp, &wctx);
    int t, g;
    uint32_t mcount = 0;
    bool ok = true;
    while (ok && ti.next(t, g)) {
      const int4 tile = p.tiles[t];
      const int s = mcount & 1;
      if (!warp_wait(&B->meta_free[s], ((mcount >> 1) & 1) ^ 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
      for (int rr = lane; rr < BT; rr += 32) {
        const RowMeta m = row_meta(p, tile, g, rr);
        DqRow d;
        d.lo = m.lo;
        d.hi = m.hi;
        d.rec = m.rec;
        d.valid = m.valid ? 1 : 0;
        d.l2 = INFINITY;
        d.dl = 0.f;
        if (m.valid) {
          const float L = lse[m.qrow];
          d.l2 = (L == -INFINITY) ? INFINITY : L * kLog2e;
          d.dl = delta[m.qrow];
        }
        meta[s * 128 + rr] = d;
      }
      warp_arrive(&B->meta_ready[s]);
      ++mcount;
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= 4 && warp < 12) {
    const int hf = (warp - 4) >> 2;           // warpgroup: keys 64hf..64hf+63 of every key tile
    const uint32_t lane_addr = uint32_t((warp & 3) << 5) << 16;
    const uint32_t tdP = tmem + lane_addr + 256;
    const int r = ((warp & 3) << 5) + lane;
    const float scale_log2 = scale * kLog2e;
    TileIter ti;
    ti.init(&p, w, &B->ring, kClaimWarp, &wctx);
    int t, g;
    uint32_t kv_count = 0, dp_cnt = 0, mcount = 0;
    bool ok = true;
    while (ok && ti.next(t, g)) {
      const int4 tile = p.tiles[t];
      const int n_kt = (tile.w - tile.z + BT - 1) / BT;
      const int ms = mcount & 1;
      if (!warp_wait(&B->meta_ready[ms], (mcount >> 1) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
      const DqRow m = meta[ms * 128 + r];
      warp_arrive(&B->meta_free[ms]);
      ++mcount;
      const float l2 = m.l2, dl = m.dl;
      for (int j = 0; j < n_kt; ++j) {
        const uint32_t c = kv_count + j;
        const int s = c & 1;
        if (!warp_wait(&B->s_ready[s], (c >> 1) & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
        if (!warp_wait(&B->dp_ready, dp_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
        ++dp_cnt;
        tc_fence_after();
        const uint32_t tS = tmem + lane_addr + s * 128;
        const int k0 = tile.z + j * BT;
        const int a = m.lo - k0, b = m.hi - k0;   // the row's allowed columns of this key tile
        // warp-uniform choice: both paths issue warp-collective tcgen05.ld/st
        if (__all_sync(0xffffffffu, a <= hf * 64 && b >= hf * 64 + 64))
          ds_tile<false>(tS, tdP, hf, a, b, scale_log2, l2, dl);
        else
          ds_tile<true>(tS, tdP, hf, a, b, scale_log2, l2, dl);
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(&B->ds_ready);
      }
      if (!ok) break;
      kv_count += n_kt;
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= 12) {
    // epilogue warps 12-15: warp 12 + q stores rows 32q..32q+31 (TMEM lanes) of each
    // tile's dQ, all D columns, as the (chunk, block) entries' dq partials; dQ is
    // released to the MMA thread after its last TMEM read
    const int r = ((warp & 3) << 5) + lane;
    const uint32_t tdQ = tmem + (uint32_t((warp & 3) << 5) << 16) + 384;
    float* scratch = reinterpret_cast<float*>(smem + Dm::kOffScratch) + (warp - 12) * 512;
    TileIter ti;
    ti.init(&p, w, &B->ring, kClaimWarp, &wctx);
    int t, g;
    uint32_t dq_cnt = 0;
    bool ok = true;
    while (ok && ti.next(t, g)) {
      const int4 tile = p.tiles[t];
      const RowMeta m = row_meta(p, tile, g, r);
      if (!warp_wait(&B->dq_ready, dq_cnt & 1, wctx, 2 * 10000 + __LINE__)) { ok = false; break; }
      ++dq_cnt;
      tc_fence_after();
      // the warp's 32 rows are 32/G whole tokens of one block, all G heads of KV head g
      // (valid is warp-uniform when bulk stores are used)
      const int z0 = __shfl_sync(0xffffffffu, m.valid ? m.rec / p.Hq : 0, 0);
      const bool wv = __shfl_sync(0xffffffffu, m.valid ? 1 : 0, 0) != 0;
      if (p.partial_bf16) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tdQ + cc * 32, v);
          tmem_wait_ld();
          reg_fence<32>(v);
          if (cc == D / 32 - 1) {   // dQ read: the next tile's first dQ += dS K may start
            tc_fence_before();
            warp_arrive(&B->dq_free);
          }
          if (bulk)
            warp_bulk_store32_bf16<0>(scratch, v, scale, &tm_dq, cc * 32, g * p.G, z0, wv);
          else if (m.valid)
            lane_store32_bf16(static_cast<uint16_t*>(dq_part) + size_t(m.rec) * D + cc * 32, v, scale);
          __syncwarp();   // m.valid differs across the warp's rows: converge before the next tcgen05.ld
        }
      } else if (bulk) {
#pragma unroll 1
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tdQ + cc * 16, v);
          tmem_wait_ld();
          reg_fence<16>(v);
          if (cc == D / 16 - 1) {
            tc_fence_before();
            warp_arrive(&B->dq_free);
          }
          warp_bulk_store16<0>(scratch, v, scale, &tm_dq, cc * 16, g * p.G, z0, wv);
        }
      } else {
        float* dst = static_cast<float*>(dq_part) + size_t(m.rec) * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tdQ + cc * 16, v);
          tmem_wait_ld();
          reg_fence<16>(v);
          if (cc == D / 16 - 1) {
            tc_fence_before();
            warp_arrive(&B->dq_free);
          }
          warp_store_rows<16>(scratch, reinterpret_cast<const float*>(v), scale, m.valid ? dst + cc * 16 : nullptr);
        }
      }
    }
    // bulk stores of this warp complete before the CTA exits
    if (lane == 0) bulk_wait0();
    __syncwarp();
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
  if (tid == 0) p.timers[(p.W + p.Wb + w) * 2 + 1] = global_timer_ns();
}

}  // namespace

bool bwd_sm100_supported(const DevPlan& p) {
  const int rows = p.G * p.bs;
  return (p.d == 64 || p.d == 128) && rows % 8 == 0 && rows <= BT && tensor_maps_available();
}

namespace {

template <int D>
cudaError_t launch_bwd_sm100(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const uint16_t* dout, const float* lse, const float* delta, float scale, float* dk,
                             float* dv, void* dq_part, cudaStream_t s, int which) {
  constexpr uint32_t kSmem = Dims<D>::kSmemBytes;
  CUtensorMap tq, tdo, tk, tv, tdk, tdv, tdq;
  if (!make_bf16_map_3d(&tq, q, D, p.Hq, p.Nq, p.G, p.bs) || !make_bf16_map_3d(&tdo, dout, D, p.Hq, p.Nq, p.G, p.bs) ||
      !make_bf16_map_3d(&tk, k, D, p.Hkv, p.N, 1, BT) || !make_bf16_map_3d(&tv, v, D, p.Hkv, p.N, 1, BT) ||
      !make_f32_map_3d(&tdk, dk, D, p.Hkv, p.N, 16, 1, 32) || !make_f32_map_3d(&tdv, dv, D, p.Hkv, p.N, 16, 1, 32))
    return cudaErrorInvalidValue;
  // dq partial records by bulk stores when a warp's 32 rows are 32/G whole tokens of one block
  const bool bulk_dq = 32 % p.G == 0 && (p.G * p.bs) % 32 == 0 && p.E > 0;
  if (bulk_dq) {
    const bool ok = p.partial_bf16
                        ? make_bf16_store_map_3d(&tdq, dq_part, D, p.Hq, uint64_t(p.E) * p.bs, p.G, 32 / p.G)
                        : make_f32_map_3d(&tdq, dq_part, D, p.Hq, uint64_t(p.E) * p.bs, 16, p.G, 32 / p.G);
    if (!ok) return cudaErrorInvalidValue;
  } else {
    memset(&tdq, 0, sizeof(tdq));
  }
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmem));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
  if (e != cudaSuccess) return e;
  // run-time claims start from item 0 at every launch (each kernel its own cursor)
  if (which != 2) {
    if (p.dynamic && (e = cudaMemsetAsync(p.claim + 1, 0, sizeof(int), s)) != cudaSuccess) return e;
    bwd_dkdv_sm100_kernel<D><<<p.Wb, kThreads, kSmem, s>>>(tq, tdo, tk, tv, tdk, tdv, p, lse, delta, scale, dk, dv);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (which != 1) {
    if (p.dynamic && (e = cudaMemsetAsync(p.claim + 2, 0, sizeof(int), s)) != cudaSuccess) return e;
    bwd_dq_sm100_kernel<D><<<p.W, kDqThreads, kSmem, s>>>(tq, tdo, tk, tv, tdq, p, lse, delta, scale,
                                                        bulk_dq ? 1 : 0, dq_part);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

cudaError_t launch_bwd_partial_sm100(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     const uint16_t* dout, const float* lse, const float* delta, float scale,
                                     float* dk, float* dv, void* dq_part, cudaStream_t s, int which) {
  if (p.d == 64) return launch_bwd_sm100<64>(p, q, k, v, dout, lse, delta, scale, dk, dv, dq_part, s, which);
  return launch_bwd_sm100<128>(p, q, k, v, dout, lse, delta, scale, dk, dv, dq_part, s, which);
}

}  // namespace splitkv
