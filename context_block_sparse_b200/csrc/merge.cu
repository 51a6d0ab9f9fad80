// HBM-bound kernels around the partial-attention kernels:
//   merge_kernel        exact log-sum-exp combine of a block's chunk records plus
//                       its in-block term -> o, lse
//   delta_kernel        Delta_i = dout_i . o_i (backward preamble)
//   bwd_reduce_kernel   dq = the in-block term's dq + the chunk dq partials
//                       (ascending chunk); dkb, dvb of the in-block term
//
// News page "Split-KV speeds diffusion drafter training by keeping long-context
// data local", section "Exchange the smaller side" (partials combined exactly
// with their normalisation statistics) and section "Why short queries change
// the problem" (every block also attends to all tokens inside itself; those
// bs keys are the draft block's own kb/vb rows).
//
// One CTA per (block b, KV head g) handles the G*bs query rows (G heads x bs
// tokens) that read the same bs block keys, four threads per row (see the row
// layout below).  All loops run in a fixed order, so results are deterministic.
#include <cfloat>

#include "common.cuh"
#include "splitkv_internal.h"

namespace splitkv {
namespace {

constexpr int kMergeThreads = 256;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int DPL>
__device__ __forceinline__ void load_bf16_row(const uint16_t* src, float (&x)[DPL]) {
  if constexpr (DPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(src);
    x[0] = __uint_as_float(u << 16);
    x[1] = __uint_as_float(u & 0xffff0000u);
  }
}

template <int DPL>
__device__ __forceinline__ void load_f32_row(const float* src, float (&x)[DPL]) {
  if constexpr (DPL == 4) {
    const float4 u = *reinterpret_cast<const float4*>(src);
    x[0] = u.x;
    x[1] = u.y;
    x[2] = u.z;
    x[3] = u.w;
  } else {
    const float2 u = *reinterpret_cast<const float2*>(src);
    x[0] = u.x;
    x[1] = u.y;
  }
}

// ---------------------------------------------------------------------------
// Row layout of the merge and reduce kernels: four threads (a quad) per query
// row; thread u of the quad owns the 16-byte fp32 granules u, u + 4, u + 8, ...
// of the row (NG = D / 16 of them, 4 * NG dimensions), so one load instruction
// of a warp reads 8 rows x 64 contiguous bytes.  Dot products over the row are
// quad sums (two shuffles).  The block's chunk entries are staged in shared
// memory kEStage at a time.
// ---------------------------------------------------------------------------
constexpr int kEStage = 512;
constexpr int kRowsPerPass = kMergeThreads / 4;

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// the thread's dimensions of a bf16 row: granule k covers dims 4 (u + 4k) .. +3
template <int NG>
__device__ __forceinline__ void load_bf16_quad(const uint16_t* row, int u, float (&x)[NG][4]) {
#pragma unroll
  for (int k = 0; k < NG; ++k) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 4 * (u + 4 * k));
    x[k][0] = __uint_as_float(w.x << 16);
    x[k][1] = __uint_as_float(w.x & 0xffff0000u);
    x[k][2] = __uint_as_float(w.y << 16);
    x[k][3] = __uint_as_float(w.y & 0xffff0000u);
  }
}

template <int NG>
__device__ __forceinline__ void load_f32_quad(const float* row, int u, float4 (&x)[NG]) {
#pragma unroll
  for (int k = 0; k < NG; ++k) x[k] = __ldg(reinterpret_cast<const float4*>(row + 4 * (u + 4 * k)));
}

// Record rows of either element type, held as raw 32-bit words until use: a
// granule (4 dimensions) is RW words -- 4 for float32, 2 for bf16 pairs -- so
// that bf16 records keep twice as many entries in flight in the same registers.
template <bool kBf16>
struct Rec {
  static constexpr int RW = kBf16 ? 2 : 4;
  template <int NG>
  __device__ __forceinline__ static void load(const void* base, size_t row, int u, uint32_t (&x)[NG][RW]) {
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      if constexpr (kBf16) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + row + 4 * (u + 4 * k)));
        x[k][0] = w.x;
        x[k][1] = w.y;
      } else {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const float*>(base) + row + 4 * (u + 4 * k)));
        x[k][0] = w.x;
        x[k][1] = w.y;
        x[k][2] = w.z;
        x[k][3] = w.w;
      }
    }
  }
  __device__ __forceinline__ static float4 get(const uint32_t (&x)[RW]) {
    if constexpr (kBf16)
      return make_float4(__uint_as_float(x[0] << 16), __uint_as_float(x[0] & 0xffff0000u),
                         __uint_as_float(x[1] << 16), __uint_as_float(x[1] & 0xffff0000u));
    else
      return make_float4(__uint_as_float(x[0]), __uint_as_float(x[1]), __uint_as_float(x[2]), __uint_as_float(x[3]));
  }
  template <int NG>
  __device__ __forceinline__ static void zero(uint32_t (&x)[NG][RW]) {
#pragma unroll
    for (int k = 0; k < NG; ++k)
#pragma unroll
      for (int i = 0; i < RW; ++i) x[k][i] = 0u;
  }
};

// Stage entries [c0, c0 + cnt) of the block into sE (whole CTA; barriers inside).
__device__ __forceinline__ void stage_entries(int* sE, const int* __restrict__ entries, int c0, int cnt) {
  __syncthreads();
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) sE[i] = entries[c0 + i];
  __syncthreads();
}

// Rows of block b under a MergeDest: the owner's index (into dest.o / dest.lse) and the
// block's first row in the owner's [R][rows_owner] receive buffer, at slot dest.self.
// ok = false only if the owner formula failed; then nothing is stored and the status
// word records it.
__device__ __forceinline__ int dest_of_block(const DevPlan& p, const MergeDest& dest, int b, size_t& row_base,
                                             bool& ok) {
  const int own = int((int64_t(b + 1) * dest.R - 1) / p.A);
  const int lo = int(int64_t(own) * p.A / dest.R), hi = int(int64_t(own + 1) * p.A / dest.R);
  ok = own >= 0 && own < dest.R && b >= lo && b < hi && dest.self >= 0 && dest.self < dest.R;
  row_base = ok ? size_t(dest.self) * size_t(hi - lo) * p.bs + size_t(b - lo) * p.bs : 0;
  if (!ok && threadIdx.x == 0) atomicCAS(p.status, 0, SPLITKV_ERR_INVALID_ARG);
  return ok ? own : 0;
}

// ---------------------------------------------------------------------------
// Helpers of the merge and reduce kernels.  The reduce kernel runs two roles of
// 128 threads: the stream role reads the block's chunk records (the HBM-bound part)
// 32 rows at a time, a quad per row; the block role computes the in-block term of
// the same rows (bs keys of the block itself) and hands it over per pass of 32 rows
// through one of two shared-memory slots: "full" (block -> stream) and "empty"
// (stream -> block, before the slot's next use two passes later) are named barriers
// over both roles.
// ---------------------------------------------------------------------------
constexpr int kRoleThreads = kMergeThreads / 2;
constexpr int kRoleRows = kRoleThreads / 4;   // rows of one pass (a quad per row in the stream role)
constexpr int kBarStream = 1, kBarBlock = 2, kBarFull = 3, kBarEmpty = 5;   // full / empty: + slot

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~size_t(15); }

// float4 granule gi of row rl in a [32][D] fp32 slot; rows rl and rl ^ 1 use opposite
// halves of the banks for the same granule, so a quad's 16-byte accesses from two rows
// (one 128-byte wavefront) never share a bank.
template <int D>
__device__ __forceinline__ int slot_off(int rl, int gi) {
  return rl * D + 4 * (gi ^ ((rl & 1) << 2));
}

template <int kSlot>
__device__ __forceinline__ void slot_handoff_wait(int j) {   // block role: slot kSlot free again
  if (j >= 2) named_sync<kBarEmpty + kSlot>(kMergeThreads);
}

__device__ __forceinline__ void slot_full_arrive(int sl) {
  sl ? named_arrive<kBarFull + 1>(kMergeThreads) : named_arrive<kBarFull>(kMergeThreads);
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
  return x;
}

// Stage the block's keys and values into shared memory, 16-byte chunks, by the
// nthr threads from t0 on (swizzled for ldmatrix when kSwz).
template <int D, bool kSwz>
__device__ __forceinline__ void stage_block_rows(const DevPlan& p, int b, int g, const uint16_t* __restrict__ kb,
                                                 const uint16_t* __restrict__ vb, uint16_t* sKb, uint16_t* sVb,
                                                 int t0, int nthr) {
  const int gt = threadIdx.x - t0, bs = p.bs;
  for (int idx = gt; idx < bs * (D / 8); idx += nthr) {
    const int t = idx / (D / 8), ch = idx % (D / 8);
    const size_t src = (size_t(b * bs + t) * p.Hkv + g) * D + ch * 8;
    const int dst = kSwz ? swz<D>(t, ch) : t * D + ch * 8;
    *reinterpret_cast<uint4*>(sKb + dst) = *reinterpret_cast<const uint4*>(kb + src);
    *reinterpret_cast<uint4*>(sVb + dst) = *reinterpret_cast<const uint4*>(vb + src);
  }
}
// Stage the rows' q (or dout) into a swizzled [rows][D] tile, by the nthr threads
// from t0 on.
template <int D>
__device__ __forceinline__ void stage_query_rows(const DevPlan& p, int b, int g, const uint16_t* __restrict__ src_rows,
                                                 uint16_t* sRows, int t0, int nthr) {
  const int gt = threadIdx.x - t0, bs = p.bs, R = p.G * bs;
  for (int idx = gt; idx < R * (D / 8); idx += nthr) {
    const int r = idx / (D / 8), ch = idx % (D / 8);
    const int tt = r / p.G, hh = r - tt * p.G;
    const size_t src = (size_t(b * bs + tt) * p.Hq + g * p.G + hh) * D + ch * 8;
    *reinterpret_cast<uint4*>(sRows + swz<D>(r, ch)) = *reinterpret_cast<const uint4*>(src_rows + src);
  }
}

// ---------------------------------------------------------------------------
// merge: grid (A, Hkv), all 256 threads; a CTA combines the G * bs rows of block b
// under KV head g, 64 rows a pass, a quad per row.  Per row: the in-block term --
// online softmax over the bs block keys: M_in (base 2), L_in and the unnormalised
// acc_in = sum_k 2^(s_k - M_in) v_k -- then the chunk records in ascending chunk
// order (EG in flight) with an online reference maximum M: acc += l_c 2^(m_c - M) O_c,
// L += l_c 2^(m_c - M); o = acc / L, lse = (M + log2 L) ln 2.
// When rows and block keys come in multiples of 16 the in-block term of every row
// is computed first, on the tensor cores (mma.sync; P rounded to bf16 for P V, as in
// the chunk kernels), into shared memory, and each row's pass starts from it; other
// shapes compute it per row on the FMA pipes in fp32.
// smem: kb, vb [bs][D] bf16 | entry ids [kEStage] | tensor path: q rows [rows][D] bf16,
// in-block acc [rows][D] fp32, (M_in, L_in) [rows] float2; tensor-path bf16 tiles swizzled.
// ---------------------------------------------------------------------------
struct MergeSmem {
  size_t kb, vb, e, qr, ib, ml, total;
};
__host__ __device__ inline MergeSmem merge_smem(int D, int bs, int R, bool tc) {
  MergeSmem L;
  size_t o = 0;
  L.kb = o;
  o += al16(size_t(bs) * D * 2);
  L.vb = o;
  o += al16(size_t(bs) * D * 2);
  L.e = o;
  o += al16(size_t(kEStage) * 4);
  L.qr = o;
  o += al16(tc ? size_t(R) * D * 2 : 0);
  L.ib = o;
  o += al16(tc ? size_t(R) * D * 4 : 0);
  L.ml = o;
  o += al16(tc ? size_t(R) * 8 : 0);
  L.total = o;
  return L;
}

// In-block term of every row on the tensor cores: task t = (16-row tile t >> 1, half
// t & 1 of the head dim), tasks spread over the 8 warps.  S = Q K^T over 16 block keys
// at a time, an online maximum per row (quad max), P = 2^(s - M) and the half's
// acc += P V.  Fragment layouts of m16n8k16: element e of an accumulator n-tile is row
// gq + 8 (e >> 1), column 2 tq + (e & 1).  Results: sIb rows (slot_off layout), sML.
template <int D>
__device__ __forceinline__ void merge_block_tc(const DevPlan& p, float scale_log2, const uint16_t* sKb,
                                               const uint16_t* sVb, const uint16_t* sQr, float* sIb, float2* sML) {
  constexpr int kNH = D / 16;   // 8-column n-tiles in half the head dim
  const int bs = p.bs, R = p.G * bs;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  for (int task = w; task < 2 * (R / 16); task += kMergeThreads / 32) {
    const int r0 = (task >> 1) * 16, dh = task & 1;
    float acc[kNH][4];
#pragma unroll
    for (int nn = 0; nn < kNH; ++nn)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nn][e] = 0.f;
    float M[2] = {-INFINITY, -INFINITY}, L[2] = {0.f, 0.f};   // rows gq, gq + 8 (L: this thread's columns)
    for (int kc = 0; kc < bs; kc += 16) {
      float s[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t qa[4], kf[4];
        ldsm_x4(qa[0], qa[1], qa[2], qa[3], sQr + swz<D>(r0 + (lane & 15), 2 * ks + (lane >> 4)));
        ldsm_x4(kf[0], kf[1], kf[2], kf[3],
                sKb + swz<D>(kc + (lane & 7) + ((lane >> 4) << 3), 2 * ks + ((lane >> 3) & 1)));
        mma_bf16_16816(s[0], qa, kf[0], kf[1]);
        mma_bf16_16816(s[1], qa, kf[2], kf[3]);
      }
      uint32_t pa[4];   // word 2 nt + h: row gq + 8h, keys kc + 8 nt + 2 tq and + 1
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float x[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = s[c >> 1][2 * h + (c & 1)] * scale_log2;
        const float mn = fmaxf(M[h], quad_max(fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]))));
        const float corr = fast_exp2(M[h] - mn);   // 0 on the first keys (M = -inf)
        M[h] = mn;
        float e4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) e4[c] = fast_exp2(x[c] - mn);
        L[h] = L[h] * corr + ((e4[0] + e4[1]) + (e4[2] + e4[3]));
#pragma unroll
        for (int nn = 0; nn < kNH; ++nn) {
          acc[nn][2 * h] *= corr;
          acc[nn][2 * h + 1] *= corr;
        }
        pa[h] = pack_bf16(e4[0], e4[1]);
        pa[2 + h] = pack_bf16(e4[2], e4[3]);
      }
#pragma unroll
      for (int nn = 0; nn < kNH; nn += 2) {   // acc (the task's columns) += P V
        const int kr = kc + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ch = dh * (D / 16) + nn + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, sVb + swz<D>(kr, ch));
        mma_bf16_16816(acc[nn], pa, b0, b1);
        mma_bf16_16816(acc[nn + 1], pa, b2, b3);
      }
    }
#pragma unroll
    for (int nn = 0; nn < kNH; ++nn)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = r0 + gq + 8 * h;
        const int col = dh * (D / 2) + nn * 8 + 2 * tq;
        *reinterpret_cast<float2*>(sIb + slot_off<D>(r, col >> 2) + (col & 3)) =
            make_float2(acc[nn][2 * h], acc[nn][2 * h + 1]);
      }
    if (dh == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float l = quad_sum(L[h]);
        if (tq == 0) sML[r0 + gq + 8 * h] = make_float2(M[h], l);
      }
    }
  }
}

template <int D, bool kBf16Rec, bool kTC>
__global__ void __launch_bounds__(kMergeThreads, 2)
    merge_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ kb,
                 const uint16_t* __restrict__ vb, float scale_log2, const void* __restrict__ part_o,
                 const float* __restrict__ part_m, const float* __restrict__ part_l, void* __restrict__ o,
                 int o_bf16, float* __restrict__ lse, const MergeDest dest) {
  constexpr int NG = D / 16;
  using RecT = Rec<kBf16Rec>;
  constexpr int EG = 64 / (NG * RecT::RW);   // entries whose records are in flight together
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int bs = p.bs, R = p.G * bs;
  const MergeSmem S = merge_smem(D, bs, R, kTC);
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw + S.kb);
  uint16_t* sVb = reinterpret_cast<uint16_t*>(smem_raw + S.vb);
  int* sE = reinterpret_cast<int*>(smem_raw + S.e);
  float* sIb = reinterpret_cast<float*>(smem_raw + S.ib);
  float2* sML = reinterpret_cast<float2*>(smem_raw + S.ml);
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, u = tid & 3;
  const bool bterm = p.block_term && b >= p.bt_lo && b < p.bt_hi;   // in-block term of this block here
  for (int idx = tid; bterm && idx < bs * (D / 8); idx += kMergeThreads) {
    const int t = idx / (D / 8), ch = idx % (D / 8);
    const size_t src = (size_t(b * bs + t) * p.Hkv + g) * D + ch * 8;
    const int dst = kTC ? swz<D>(t, ch) : t * D + ch * 8;
    *reinterpret_cast<uint4*>(sKb + dst) = *reinterpret_cast<const uint4*>(kb + src);
    *reinterpret_cast<uint4*>(sVb + dst) = *reinterpret_cast<const uint4*>(vb + src);
  }
  if constexpr (kTC) {
    if (bterm) {
      uint16_t* sQr = reinterpret_cast<uint16_t*>(smem_raw + S.qr);
      for (int idx = tid; idx < R * (D / 8); idx += kMergeThreads) {
        const int r = idx / (D / 8), ch = idx % (D / 8);
        const int tt = r / p.G, hh = r - tt * p.G;
        const size_t src = (size_t(b * bs + tt) * p.Hq + g * p.G + hh) * D + ch * 8;
        *reinterpret_cast<uint4*>(sQr + swz<D>(r, ch)) = *reinterpret_cast<const uint4*>(q + src);
      }
      __syncthreads();
      merge_block_tc<D>(p, scale_log2, sKb, sVb, sQr, sIb, sML);
    }
  }
  const int e0 = p.block_entry_ptr[b], n = p.block_entry_ptr[b + 1] - e0;
  const int n_block_keys = (bterm && !kTC) ? bs : 0;   // in-block term computed per row (FMA path)
  // output rows: the plan's own outputs, or the owner's receive buffer (see MergeDest);
  // row_base = this block's first row in the buffer written to
  void* o_out = o;
  float* lse_out = lse;
  int out_bf16 = o_bf16;
  size_t row_base = size_t(b) * bs;
  bool out_ok = true;
  if (dest.o != nullptr) {
    const int own = dest_of_block(p, dest, b, row_base, out_ok);
    o_out = dest.o[own];
    lse_out = dest.lse[own];
    out_bf16 = 0;
  }
  for (int r0 = 0; r0 < R; r0 += kRowsPerPass) {
    // rows ordered (token, head): the 8 rows of a warp are contiguous records
    const int r = min(r0 + (tid >> 2), R - 1);          // rows past R compute, never store
    const bool active = r0 + (tid >> 2) < R;
    const int tt = r / p.G, hh = r - tt * p.G;
    const int head = g * p.G + hh;
    const size_t qrow = size_t(b * bs + tt) * p.Hq + head;
    stage_entries(sE, p.block_entries + e0, 0, min(n, kEStage));   // (its barrier also publishes sIb, sML)
    float acc[NG][4];
    float M = -INFINITY, L = 0.f;
    if (kTC && bterm) {   // the row's in-block state
      const float2 ml = sML[r];
      M = ml.x;
      L = ml.y;
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        const float4 x = *reinterpret_cast<const float4*>(sIb + slot_off<D>(r, u + 4 * k));
        acc[k][0] = x.x;
        acc[k][1] = x.y;
        acc[k][2] = x.z;
        acc[k][3] = x.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < NG; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[k][i] = 0.f;
    }
    if (n_block_keys > 0) {   // in-block term per row: online softmax over the block keys (base 2)
      float qv[NG][4];
      load_bf16_quad<NG>(q + qrow * D, u, qv);
      for (int key = 0; key < n_block_keys; ++key) {
        float kv[NG][4];
        load_bf16_quad<NG>(sKb + key * D, u, kv);
        float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < NG; ++k)
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = fmaf(qv[k][i], kv[k][i], d4[i]);
        const float sc = quad_sum((d4[0] + d4[1]) + (d4[2] + d4[3])) * scale_log2;
        const float mn = fmaxf(M, sc);
        const float corr = fast_exp2(M - mn);
        const float pr = fast_exp2(sc - mn);
        L = L * corr + pr;
        float vv[NG][4];
        load_bf16_quad<NG>(sVb + key * D, u, vv);
#pragma unroll
        for (int k = 0; k < NG; ++k)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[k][i] = fmaf(pr, vv[k][i], acc[k][i] * corr);
        M = mn;
      }
    }
    // chunk records in ascending chunk order, EG in flight; online reference M
    for (int c0 = 0; c0 < n; c0 += kEStage) {
      const int cnt = min(kEStage, n - c0);
      if (c0 > 0) stage_entries(sE, p.block_entries + e0, c0, cnt);
      for (int i0 = 0; i0 < cnt; i0 += EG) {
        uint32_t ov[EG][NG][RecT::RW];
        float mx[EG], lx[EG];
#pragma unroll
        for (int v = 0; v < EG; ++v) {
          lx[v] = 0.f;
          mx[v] = -INFINITY;
          if (i0 + v < cnt) {
            const size_t rec = size_t(sE[i0 + v] * bs + tt) * p.Hq + head;
            RecT::template load<NG>(part_o, rec * D, u, ov[v]);
            const float lr = __ldg(part_l + rec), mr = __ldg(part_m + rec);
            lx[v] = lr;
            mx[v] = lr > 0.f ? mr * kLog2e : -INFINITY;
          } else {
            RecT::template zero<NG>(ov[v]);
          }
        }
        float mg = mx[0];
#pragma unroll
        for (int v = 1; v < EG; ++v) mg = fmaxf(mg, mx[v]);
        if (mg > M) {
          const float f = fast_exp2(M - mg);
#pragma unroll
          for (int k = 0; k < NG; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[k][i] *= f;
          L *= f;
          M = mg;
        }
#pragma unroll
        for (int v = 0; v < EG; ++v) {
          const float wv = lx[v] > 0.f ? lx[v] * fast_exp2(mx[v] - M) : 0.f;
          L += wv;
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const float4 x = RecT::get(ov[v][k]);
            acc[k][0] = fmaf(wv, x.x, acc[k][0]);
            acc[k][1] = fmaf(wv, x.y, acc[k][1]);
            acc[k][2] = fmaf(wv, x.z, acc[k][2]);
            acc[k][3] = fmaf(wv, x.w, acc[k][3]);
          }
        }
      }
    }
    if (active && out_ok) {
      const size_t orow = (row_base + tt) * p.Hq + head;   // = qrow for the plan's own outputs
      const float inv = L > 0.f ? 1.f / L : 0.f;
      if (out_bf16) {
        uint16_t* dst = static_cast<uint16_t*>(o_out) + orow * D;
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          uint2 w;
          w.x = pack_bf16(acc[k][0] * inv, acc[k][1] * inv);
          w.y = pack_bf16(acc[k][2] * inv, acc[k][3] * inv);
          *reinterpret_cast<uint2*>(dst + 4 * (u + 4 * k)) = w;
        }
      } else {
        float* dst = static_cast<float*>(o_out) + orow * D;
#pragma unroll
        for (int k = 0; k < NG; ++k)
          *reinterpret_cast<float4*>(dst + 4 * (u + 4 * k)) =
              make_float4(acc[k][0] * inv, acc[k][1] * inv, acc[k][2] * inv, acc[k][3] * inv);
      }
      if (u == 0) lse_out[orow] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// Delta = rowsum(dout * o): one warp per (token, head) row
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    delta_kernel(int rows, const void* __restrict__ o, int o_bf16, const uint16_t* __restrict__ dout,
                 float* __restrict__ delta) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int warps_total = (gridDim.x * blockDim.x) >> 5;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps_total) {
    float dv[DPL], ov[DPL];
    load_bf16_row<DPL>(dout + size_t(r) * D + lane * DPL, dv);
    if (o_bf16) {
      load_bf16_row<DPL>(static_cast<const uint16_t*>(o) + size_t(r) * D + lane * DPL, ov);
    } else {
      load_f32_row<DPL>(static_cast<const float*>(o) + size_t(r) * D + lane * DPL, ov);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) s = fmaf(dv[i], ov[i], s);
    s = warp_sum(s);
    if (lane == 0) delta[r] = s;
  }
}

// ---------------------------------------------------------------------------
// dq reduce + in-block backward: grid (A, Hkv); a CTA handles the G * bs rows of
// block b under KV head g: dq = the in-block term's dq + the chunk dq partials in
// ascending chunk order; dkb, dvb of the in-block term.  Two kernels:
//
//  bwd_reduce_tc_kernel (rows and block keys in multiples of 16): all 256 threads.
//    First the in-block term of every row on the tensor cores (mma.sync m16n8k16:
//    bf16 operands, P and dS rounded to bf16 as in the chunk kernels; fp32
//    accumulators), its dq into shared memory; then 64 rows a pass, a quad per row,
//    dq = that + the partials (EG records in flight per thread); last dkb = scale dS^T Q
//    and dvb = P^T dO from P, dS kept in shared memory.
//
//  bwd_reduce_kernel (any shape): the two roles above run side by side -- the
//    stream role sums the partials of 32 rows a pass and adds the slot's in-block dq;
//    the block role computes P, dS and the in-block dq on the FMA pipes in fp32 (a quad
//    per row), then dkb, dvb (a warp per pair of block keys).
// ---------------------------------------------------------------------------
// Shared memory of bwd_reduce_kernel (byte offsets, 16-byte aligned):
//   slot   [2][32][D] fp32    in-block dq of a pass, block role -> stream role
//   kb, vb [bs][D] bf16       the block's keys and values
//   p, ds  [rows][bs] fp32
//   e      [kEStage] int      entry ids (stream role)
//   qr, dr [rows][D] bf16     the rows' q and dout (when stage_rows)
// rows = G * bs ordered (token, head).
struct ReduceSmem {
  size_t slot, kb, vb, p, ds, e, qr, dr, total;
};
__host__ __device__ inline ReduceSmem reduce_smem(int D, int bs, int R, bool stage_rows) {
  ReduceSmem L;
  size_t o = 0;
  L.slot = o;
  o += al16(size_t(2) * kRoleRows * D * 4);
  L.kb = o;
  o += al16(size_t(bs) * D * 2);
  L.vb = o;
  o += al16(size_t(bs) * D * 2);
  L.p = o;
  o += al16(size_t(R) * bs * 4);
  L.ds = o;
  o += al16(size_t(R) * bs * 4);
  L.e = o;
  o += al16(size_t(kEStage) * 4);
  const size_t rows = stage_rows ? size_t(R) * D * 2 : 0;
  L.qr = o;
  o += al16(rows);
  L.dr = o;
  o += al16(rows);
  L.total = o;
  return L;
}

// Shared memory of bwd_reduce_tc_kernel: kb, vb [bs][D] and qr, dr [rows][D] bf16
// (swizzled for ldmatrix); p, ds [rows][bs + 8] bf16 (the pad keeps ldmatrix rows on
// distinct banks); ib [rows][D] fp32 in-block dq (slot_off layout); entry ids.
struct ReduceTcSmem {
  size_t kb, vb, qr, dr, p, ds, ib, e, total;
};
__host__ __device__ inline ReduceTcSmem reduce_tc_smem(int D, int bs, int R) {
  ReduceTcSmem L;
  size_t o = 0;
  L.kb = o;
  o += al16(size_t(bs) * D * 2);
  L.vb = o;
  o += al16(size_t(bs) * D * 2);
  L.qr = o;
  o += al16(size_t(R) * D * 2);
  L.dr = o;
  o += al16(size_t(R) * D * 2);
  L.p = o;
  o += al16(size_t(R) * (bs + 8) * 2);
  L.ds = o;
  o += al16(size_t(R) * (bs + 8) * 2);
  L.ib = o;
  o += al16(size_t(R) * D * 4);
  L.e = o;
  o += al16(size_t(kEStage) * 4);
  L.total = o;
  return L;
}

struct BlockIO {   // global operands of the block role
  const uint16_t* q;
  const uint16_t* kb;
  const uint16_t* vb;
  const uint16_t* dout;
  const float* lse;
  const float* delta;
  float scale;
  float* dkb;
  float* dvb;
};

// Block role on the FMA pipes (any rows / block keys): a quad per row for P, dS and
// the in-block dq; a warp per pair of block keys for dkb, dvb.
template <int D>
__device__ __forceinline__ void block_role_fma(const DevPlan& p, int b, int g, const BlockIO& io, int stage_rows,
                                               float* sSlot, uint16_t* sKb, uint16_t* sVb, float* sP, float* sdS,
                                               uint16_t* sQr, uint16_t* sDr) {
  constexpr int NG = D / 16;
  constexpr int DPL = D / 32;
  const int bs = p.bs, R = p.G * bs;
  const int gt = threadIdx.x - kRoleThreads, u = gt & 3, rl = gt >> 2, bwarp = gt >> 5, lane = threadIdx.x & 31;
  stage_block_rows<D, false>(p, b, g, io.kb, io.vb, sKb, sVb, kRoleThreads, kRoleThreads);
  named_sync<kBarBlock>(kRoleThreads);
  const float scale_log2 = io.scale * kLog2e;
  const int npass = (R + kRoleRows - 1) / kRoleRows;
  for (int j = 0; j < npass; ++j) {
    const int r = min(j * kRoleRows + rl, R - 1);
    const bool active = j * kRoleRows + rl < R;
    const int tt = r / p.G, hh = r - tt * p.G;
    const size_t qrow = size_t(b * bs + tt) * p.Hq + g * p.G + hh;
    float acc[NG][4];
    {
      float qv[NG][4], dov[NG][4];
      load_bf16_quad<NG>(io.q + qrow * D, u, qv);
      load_bf16_quad<NG>(io.dout + qrow * D, u, dov);
      const float l2 = io.lse[qrow] * kLog2e;
      const float dl = io.delta[qrow];
#pragma unroll
      for (int k = 0; k < NG; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[k][i] = 0.f;
#pragma unroll 1
      for (int key = 0; key < bs; ++key) {
        // four partial sums per dot product: dependent chains of NG, not 4 * NG, FMAs
        float sd4[4] = {0.f, 0.f, 0.f, 0.f}, dp4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          float kv[1][4], vv[1][4];
          load_bf16_quad<1>(sKb + key * D + 16 * k, u, kv);
          load_bf16_quad<1>(sVb + key * D + 16 * k, u, vv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            sd4[i] = fmaf(qv[k][i], kv[0][i], sd4[i]);
            dp4[i] = fmaf(dov[k][i], vv[0][i], dp4[i]);
          }
        }
        const float sd = quad_sum((sd4[0] + sd4[1]) + (sd4[2] + sd4[3]));
        const float dp = quad_sum((dp4[0] + dp4[1]) + (dp4[2] + dp4[3]));
        const float pr = (l2 == -INFINITY) ? 0.f : fast_exp2(sd * scale_log2 - l2);
        const float ds = pr * (dp - dl);
        if (active && u == 0) {
          sP[r * bs + key] = pr;
          sdS[r * bs + key] = ds;
        }
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          float kv[1][4];
          load_bf16_quad<1>(sKb + key * D + 16 * k, u, kv);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[k][i] = fmaf(ds, kv[0][i], acc[k][i]);
        }
      }
      if (stage_rows && active) {   // keep q and dout of this row for the dkb / dvb pass
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          const int off = r * D + 4 * (u + 4 * k);
          *reinterpret_cast<uint2*>(sQr + off) = *reinterpret_cast<const uint2*>(io.q + qrow * D + 4 * (u + 4 * k));
          *reinterpret_cast<uint2*>(sDr + off) =
              *reinterpret_cast<const uint2*>(io.dout + qrow * D + 4 * (u + 4 * k));
        }
      }
    }
    const int sl = j & 1;
    sl ? slot_handoff_wait<1>(j) : slot_handoff_wait<0>(j);
    float* slot = sSlot + sl * kRoleRows * D;
#pragma unroll
    for (int k = 0; k < NG; ++k)
      *reinterpret_cast<float4*>(slot + slot_off<D>(rl, u + 4 * k)) =
          make_float4(io.scale * acc[k][0], io.scale * acc[k][1], io.scale * acc[k][2], io.scale * acc[k][3]);
    slot_full_arrive(sl);
  }
  named_sync<kBarBlock>(kRoleThreads);   // P, dS (and the staged rows) of every row written
  // a warp per pair of block keys (k0, k0 + 1), sharing each row's loads:
  // dkb = scale * sum_r dS[r] q_r, dvb = sum_r P[r] dout_r
  for (int k0 = 2 * bwarp; k0 < bs; k0 += 2 * (kRoleThreads / 32)) {
    const int nk = min(2, bs - k0);
    float ak[2][DPL], av[2][DPL];
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
      for (int i = 0; i < DPL; ++i) ak[x][i] = av[x][i] = 0.f;
#pragma unroll 4
    for (int r = 0; r < R; ++r) {
      float qv[DPL], dov[DPL];
      if (stage_rows) {
        load_bf16_row<DPL>(sQr + r * D + lane * DPL, qv);
        load_bf16_row<DPL>(sDr + r * D + lane * DPL, dov);
      } else {
        const int tt = r / p.G, hh = r - tt * p.G;
        const size_t qrow = size_t(b * bs + tt) * p.Hq + g * p.G + hh;
        load_bf16_row<DPL>(io.q + qrow * D + lane * DPL, qv);
        load_bf16_row<DPL>(io.dout + qrow * D + lane * DPL, dov);
      }
      const int k1 = k0 + nk - 1;   // = k0 when the pair is a single key
      const float ds0 = sdS[r * bs + k0], pr0 = sP[r * bs + k0];
      const float ds1 = sdS[r * bs + k1], pr1 = sP[r * bs + k1];
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        ak[0][i] = fmaf(ds0, qv[i], ak[0][i]);
        av[0][i] = fmaf(pr0, dov[i], av[0][i]);
        ak[1][i] = fmaf(ds1, qv[i], ak[1][i]);
        av[1][i] = fmaf(pr1, dov[i], av[1][i]);
      }
    }
    for (int x = 0; x < nk; ++x) {
      const size_t krow = size_t(b * bs + k0 + x) * p.Hkv + g;
      float* dk_dst = io.dkb + krow * D + lane * DPL;
      float* dv_dst = io.dvb + krow * D + lane * DPL;
      if constexpr (DPL == 4) {
        *reinterpret_cast<float4*>(dk_dst) =
            make_float4(io.scale * ak[x][0], io.scale * ak[x][1], io.scale * ak[x][2], io.scale * ak[x][3]);
        *reinterpret_cast<float4*>(dv_dst) = make_float4(av[x][0], av[x][1], av[x][2], av[x][3]);
      } else {
        *reinterpret_cast<float2*>(dk_dst) = make_float2(io.scale * ak[x][0], io.scale * ak[x][1]);
        *reinterpret_cast<float2*>(dv_dst) = make_float2(av[x][0], av[x][1]);
      }
    }
  }
}

// In-block term of every row on the tensor cores: task t = (16-row tile t >> 1, half
// t & 1 of the head dim), tasks spread over the 8 warps.  S = Q K^T and dP = dO V^T over
// the block keys 16 at a time (both tasks of a tile compute them), P = exp2(s c - lse2),
// dS = P (dP - Delta) in registers, the half's in-block dq += dS K -> sIb (times scale);
// the tile's P, dS (bf16) -> sPb, sdSb.  Fragment layouts of m16n8k16: element e of an
// accumulator n-tile is row gq + 8 (e >> 1), column 2 tq + (e & 1).
template <int D>
__device__ __forceinline__ void reduce_inblock_tc(const DevPlan& p, int b, int g, const BlockIO& io,
                                                  const uint16_t* sKb, const uint16_t* sVb, const uint16_t* sQr,
                                                  const uint16_t* sDr, uint16_t* sPb, uint16_t* sdSb, float* sIb) {
  constexpr int kNH = D / 16;   // 8-column n-tiles in half the head dim
  const int bs = p.bs, R = p.G * bs, SB = bs + 8;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const float scale_log2 = io.scale * kLog2e;
  for (int task = w; task < 2 * (R / 16); task += kMergeThreads / 32) {
    const int r0 = (task >> 1) * 16, dh = task & 1;
    float dqa[kNH][4];
#pragma unroll
    for (int nn = 0; nn < kNH; ++nn)
#pragma unroll
      for (int e = 0; e < 4; ++e) dqa[nn][e] = 0.f;
    float l2[2], dl[2];   // statistics of the thread's rows r0 + gq, r0 + gq + 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = r0 + gq + 8 * h, tt = r / p.G, hh = r - tt * p.G;
      const size_t qrow = size_t(b * bs + tt) * p.Hq + g * p.G + hh;
      l2[h] = io.lse[qrow] * kLog2e;
      dl[h] = io.delta[qrow];
    }
    for (int kc = 0; kc < bs; kc += 16) {
      float s[2][4], dp[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t qa[4], da[4], kf[4], vf[4];
        const int ar = r0 + (lane & 15), ach = 2 * ks + (lane >> 4);
        ldsm_x4(qa[0], qa[1], qa[2], qa[3], sQr + swz<D>(ar, ach));
        ldsm_x4(da[0], da[1], da[2], da[3], sDr + swz<D>(ar, ach));
        const int br = kc + (lane & 7) + ((lane >> 4) << 3), bch = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(kf[0], kf[1], kf[2], kf[3], sKb + swz<D>(br, bch));
        ldsm_x4(vf[0], vf[1], vf[2], vf[3], sVb + swz<D>(br, bch));
        mma_bf16_16816(s[0], qa, kf[0], kf[1]);
        mma_bf16_16816(s[1], qa, kf[2], kf[3]);
        mma_bf16_16816(dp[0], da, vf[0], vf[1]);
        mma_bf16_16816(dp[1], da, vf[2], vf[3]);
      }
      // P = exp2(s c - lse2), dS = P (dP - Delta), packed as the A operand of dS K:
      // word 2 nt + h holds row gq + 8h, keys kc + 8 nt + 2 tq and + 1
      uint32_t pa[4], sa[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float pr[2], ds[2];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            pr[c] = (l2[h] == -INFINITY) ? 0.f : fast_exp2(s[nt][2 * h + c] * scale_log2 - l2[h]);
            ds[c] = pr[c] * (dp[nt][2 * h + c] - dl[h]);
          }
          pa[2 * nt + h] = pack_bf16(pr[0], pr[1]);
          sa[2 * nt + h] = pack_bf16(ds[0], ds[1]);
        }
      if (dh == 0) {   // P, dS of the tile for dvb, dkb (one of the tile's two tasks)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int off = (r0 + gq + 8 * h) * SB + kc + 8 * nt + 2 * tq;
            *reinterpret_cast<uint32_t*>(sPb + off) = pa[2 * nt + h];
            *reinterpret_cast<uint32_t*>(sdSb + off) = sa[2 * nt + h];
          }
      }
#pragma unroll
      for (int nn = 0; nn < kNH; nn += 2) {   // in-block dq (the task's columns) += dS K
        const int kr = kc + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ch = dh * (D / 16) + nn + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, sKb + swz<D>(kr, ch));
        mma_bf16_16816(dqa[nn], sa, b0, b1);
        mma_bf16_16816(dqa[nn + 1], sa, b2, b3);
      }
    }
#pragma unroll
    for (int nn = 0; nn < kNH; ++nn)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = r0 + gq + 8 * h;
        const int col = dh * (D / 2) + nn * 8 + 2 * tq;
        *reinterpret_cast<float2*>(sIb + slot_off<D>(r, col >> 2) + (col & 3)) =
            make_float2(io.scale * dqa[nn][2 * h], io.scale * dqa[nn][2 * h + 1]);
      }
  }
}

// dkb = scale dS^T Q and dvb = P^T dO on the tensor cores, contracting over the rows,
// in items (product, 16 keys, 32 columns) spread over the 8 warps.
template <int D>
__device__ __forceinline__ void reduce_kv_tc(const DevPlan& p, int b, int g, const BlockIO& io,
                                             const uint16_t* sQr, const uint16_t* sDr, const uint16_t* sPb,
                                             const uint16_t* sdSb) {
  const int bs = p.bs, R = p.G * bs, SB = bs + 8;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int nitems = 2 * (bs / 16) * (D / 32);
  for (int it = w; it < nitems; it += kMergeThreads / 32) {
    const int prod = it & 1, rest = it >> 1, km = rest / (D / 32), ng = rest % (D / 32);
    const uint16_t* sA = prod ? sPb : sdSb;   // A = P^T or dS^T (keys x rows), stored [rows][keys]
    const uint16_t* sB = prod ? sDr : sQr;    // B = dout or q (rows x columns)
    float acc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    for (int kr0 = 0; kr0 < R; kr0 += 16) {
      uint32_t a[4];
      const int mi = lane >> 3;
      ldsm_x4_t(a[0], a[1], a[2], a[3], sA + (kr0 + (lane & 7) + (mi >> 1) * 8) * SB + km * 16 + (mi & 1) * 8);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int br = kr0 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ch = ng * 4 + np * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(b0, b1, b2, b3, sB + swz<D>(br, ch));
        mma_bf16_16816(acc[2 * np], a, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
      }
    }
    float* dst = prod ? io.dvb : io.dkb;
    const float f = prod ? 1.f : io.scale;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int key = km * 16 + gq + 8 * h;
        const int col = ng * 32 + nt * 8 + 2 * tq;
        *reinterpret_cast<float2*>(dst + (size_t(b * bs + key) * p.Hkv + g) * D + col) =
            make_float2(f * acc[nt][2 * h], f * acc[nt][2 * h + 1]);
      }
  }
}

template <int D, bool kBf16Rec>
__global__ void __launch_bounds__(kMergeThreads, 2)
    bwd_reduce_tc_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ kb,
                         const uint16_t* __restrict__ vb, const uint16_t* __restrict__ dout,
                         const float* __restrict__ lse, const float* __restrict__ delta,
                         const void* __restrict__ dq_part, float scale, float* __restrict__ dq,
                         float* __restrict__ dkb, float* __restrict__ dvb, const MergeDest dest) {
  constexpr int NG = D / 16;
  using RecT = Rec<kBf16Rec>;
  constexpr int EG = 64 / (NG * RecT::RW);   // entries whose partials are in flight together
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int bs = p.bs, R = p.G * bs;
  const ReduceTcSmem L = reduce_tc_smem(D, bs, R);
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw + L.kb);
  uint16_t* sVb = reinterpret_cast<uint16_t*>(smem_raw + L.vb);
  uint16_t* sQr = reinterpret_cast<uint16_t*>(smem_raw + L.qr);
  uint16_t* sDr = reinterpret_cast<uint16_t*>(smem_raw + L.dr);
  uint16_t* sPb = reinterpret_cast<uint16_t*>(smem_raw + L.p);
  uint16_t* sdSb = reinterpret_cast<uint16_t*>(smem_raw + L.ds);
  float* sIb = reinterpret_cast<float*>(smem_raw + L.ib);
  int* sE = reinterpret_cast<int*>(smem_raw + L.e);
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, u = tid & 3;
  const bool bterm = p.block_term && b >= p.bt_lo && b < p.bt_hi;   // in-block term of this block here
  const BlockIO io{q, kb, vb, dout, lse, delta, scale, dkb, dvb};
  if (bterm) {
    stage_block_rows<D, true>(p, b, g, kb, vb, sKb, sVb, 0, kMergeThreads);
    stage_query_rows<D>(p, b, g, q, sQr, 0, kMergeThreads);
    stage_query_rows<D>(p, b, g, dout, sDr, 0, kMergeThreads);
    __syncthreads();
    reduce_inblock_tc<D>(p, b, g, io, sKb, sVb, sQr, sDr, sPb, sdSb, sIb);
  }
  // dq rows: the plan's own dq, or the owner's receive buffer (see MergeDest; dest.o)
  float* dq_out = dq;
  size_t dq_base = size_t(b) * bs;
  bool dq_ok = true;
  if (dest.o != nullptr) dq_out = dest.o[dest_of_block(p, dest, b, dq_base, dq_ok)];
  const int e0 = p.block_entry_ptr[b], n = p.block_entry_ptr[b + 1] - e0;
  for (int r0 = 0; r0 < R; r0 += kRowsPerPass) {
    const int r = min(r0 + (tid >> 2), R - 1);          // rows past R compute, never store
    const bool active = r0 + (tid >> 2) < R;
    const int tt = r / p.G, hh = r - tt * p.G;
    const int head = g * p.G + hh;
    stage_entries(sE, p.block_entries + e0, 0, min(n, kEStage));   // (its barrier also publishes sIb)
    float4 tot[NG];
#pragma unroll
    for (int k = 0; k < NG; ++k)
      tot[k] = bterm ? *reinterpret_cast<const float4*>(sIb + slot_off<D>(r, u + 4 * k))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < n; c0 += kEStage) {
      const int cnt = min(kEStage, n - c0);
      if (c0 > 0) stage_entries(sE, p.block_entries + e0, c0, cnt);
      for (int i0 = 0; i0 < cnt; i0 += EG) {
        uint32_t pv[EG][NG][RecT::RW];
#pragma unroll
        for (int v = 0; v < EG; ++v) {
          if (i0 + v < cnt) {
            const size_t rec = size_t(sE[i0 + v] * bs + tt) * p.Hq + head;
            RecT::template load<NG>(dq_part, rec * D, u, pv[v]);
          } else {
            RecT::template zero<NG>(pv[v]);
          }
        }
#pragma unroll
        for (int v = 0; v < EG; ++v)
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const float4 x = RecT::get(pv[v][k]);
            tot[k].x += x.x;
            tot[k].y += x.y;
            tot[k].z += x.z;
            tot[k].w += x.w;
          }
      }
    }
    if (active && dq_ok) {
      float* dst = dq_out + ((dq_base + tt) * p.Hq + head) * D;   // = dq + qrow * D for the plan's own dq
#pragma unroll
      for (int k = 0; k < NG; ++k) *reinterpret_cast<float4*>(dst + 4 * (u + 4 * k)) = tot[k];
    }
  }
  // P, dS of every row were published by the pass loop's barrier
  if (bterm) reduce_kv_tc<D>(p, b, g, io, sQr, sDr, sPb, sdSb);
}

template <int D, bool kBf16Rec>
__global__ void __launch_bounds__(kMergeThreads, 2)
    bwd_reduce_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ kb,
                      const uint16_t* __restrict__ vb, const uint16_t* __restrict__ dout,
                      const float* __restrict__ lse, const float* __restrict__ delta,
                      const void* __restrict__ dq_part, float scale, float* __restrict__ dq,
                      float* __restrict__ dkb, float* __restrict__ dvb, int stage_rows, const MergeDest dest) {
  constexpr int NG = D / 16;
  using RecT = Rec<kBf16Rec>;
  constexpr int EG = 64 / (NG * RecT::RW);   // entries whose partials are in flight together
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int bs = p.bs;
  const int R = p.G * bs;
  const ReduceSmem L = reduce_smem(D, bs, R, stage_rows != 0);
  float* sSlot = reinterpret_cast<float*>(smem_raw + L.slot);
  int* sE = reinterpret_cast<int*>(smem_raw + L.e);
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x;
  const bool bterm = p.block_term && b >= p.bt_lo && b < p.bt_hi;   // in-block term of this block here
  const int npass = (R + kRoleRows - 1) / kRoleRows;

  if (tid < kRoleThreads) {
    // ---- stream role ----
    const int gt = tid, u = gt & 3, rl = gt >> 2;
    const int e0 = p.block_entry_ptr[b], n = p.block_entry_ptr[b + 1] - e0;
    // dq rows: the plan's own dq, or the owner's receive buffer (see MergeDest; dest.o)
    float* dq_out = dq;
    size_t dq_base = size_t(b) * bs;
    bool dq_ok = true;
    if (dest.o != nullptr) dq_out = dest.o[dest_of_block(p, dest, b, dq_base, dq_ok)];
    for (int j = 0; j < npass; ++j) {
      const int r = min(j * kRoleRows + rl, R - 1);        // rows past R compute, never store
      const bool active = j * kRoleRows + rl < R;
      const int tt = r / p.G, hh = r - tt * p.G;
      const int head = g * p.G + hh;
      float4 tot[NG];
#pragma unroll
      for (int k = 0; k < NG; ++k) tot[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c0 = 0; c0 < n; c0 += kEStage) {
        const int cnt = min(kEStage, n - c0);
        if (j == 0 || n > kEStage) {   // entry ids staged once when they fit
          named_sync<kBarStream>(kRoleThreads);
          for (int i = gt; i < cnt; i += kRoleThreads) sE[i] = p.block_entries[e0 + c0 + i];
          named_sync<kBarStream>(kRoleThreads);
        }
        for (int i0 = 0; i0 < cnt; i0 += EG) {
          uint32_t pv[EG][NG][RecT::RW];
#pragma unroll
          for (int v = 0; v < EG; ++v) {
            if (i0 + v < cnt) {
              const size_t rec = size_t(sE[i0 + v] * bs + tt) * p.Hq + head;
              RecT::template load<NG>(dq_part, rec * D, u, pv[v]);
            } else {
              RecT::template zero<NG>(pv[v]);
            }
          }
#pragma unroll
          for (int v = 0; v < EG; ++v)
#pragma unroll
            for (int k = 0; k < NG; ++k) {
              const float4 x = RecT::get(pv[v][k]);
              tot[k].x += x.x;
              tot[k].y += x.y;
              tot[k].z += x.z;
              tot[k].w += x.w;
            }
        }
      }
      if (bterm) {   // + the rows' in-block dq
        const int sl = j & 1;
        sl ? named_sync<kBarFull + 1>(kMergeThreads) : named_sync<kBarFull>(kMergeThreads);
        const float* slot = sSlot + sl * kRoleRows * D;
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          const float4 x = *reinterpret_cast<const float4*>(slot + slot_off<D>(rl, u + 4 * k));
          tot[k].x += x.x;
          tot[k].y += x.y;
          tot[k].z += x.z;
          tot[k].w += x.w;
        }
        if (j + 2 < npass) sl ? named_arrive<kBarEmpty + 1>(kMergeThreads) : named_arrive<kBarEmpty>(kMergeThreads);
      }
      if (active && dq_ok) {
        float* dst = dq_out + ((dq_base + tt) * p.Hq + head) * D;   // = dq + qrow * D for the plan's own dq
#pragma unroll
        for (int k = 0; k < NG; ++k) *reinterpret_cast<float4*>(dst + 4 * (u + 4 * k)) = tot[k];
      }
    }
    return;
  }

  // ---- block role ----
  if (!bterm) return;   // its keys are context keys, or the term is computed on another rank
  const BlockIO io{q, kb, vb, dout, lse, delta, scale, dkb, dvb};
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw + L.kb);
  uint16_t* sVb = reinterpret_cast<uint16_t*>(smem_raw + L.vb);
  uint16_t* sQr = reinterpret_cast<uint16_t*>(smem_raw + L.qr);
  uint16_t* sDr = reinterpret_cast<uint16_t*>(smem_raw + L.dr);
  block_role_fma<D>(p, b, g, io, stage_rows, sSlot, sKb, sVb, reinterpret_cast<float*>(smem_raw + L.p),
                    reinterpret_cast<float*>(smem_raw + L.ds), sQr, sDr);
}

template <int D, bool kBf16Rec, bool kTC>
cudaError_t merge_launch(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb, float scale,
                         const void* po, const float* pm, const float* pl, void* o, int o_bf16, float* lse,
                         cudaStream_t s, const MergeDest& dest) {
  const size_t smem = merge_smem(D, p.bs, p.G * p.bs, kTC).total;
  cudaError_t e =
      cudaFuncSetAttribute(merge_kernel<D, kBf16Rec, kTC>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  merge_kernel<D, kBf16Rec, kTC><<<dim3(p.A, p.Hkv), kMergeThreads, smem, s>>>(p, q, kb, vb, scale * kLog2e, po, pm,
                                                                                pl, o, o_bf16, lse, dest);
  return cudaGetLastError();
}

template <int D, bool kBf16Rec>
cudaError_t merge_d(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                    float scale, const void* po, const float* pm, const float* pl, void* o, int o_bf16,
                    float* lse, cudaStream_t s, const MergeDest& dest) {
  // tensor path: rows and block keys in 16s (its tiles always fit: at most 163 KB)
  if ((p.G * p.bs) % 16 == 0 && p.bs % 16 == 0)
    return merge_launch<D, kBf16Rec, true>(p, q, kb, vb, scale, po, pm, pl, o, o_bf16, lse, s, dest);
  return merge_launch<D, kBf16Rec, false>(p, q, kb, vb, scale, po, pm, pl, o, o_bf16, lse, s, dest);
}

template <int D, bool kBf16Rec>
cudaError_t reduce_d(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                     const uint16_t* dout, const float* lse, const float* delta, const void* dq_part,
                     float scale, float* dq, float* dkb, float* dvb, cudaStream_t s, const MergeDest& dest) {
  const int R = p.G * p.bs;
  constexpr size_t kMaxSmem = size_t(227) * 1024;
  // tensor path: rows and block keys in 16s, and its tiles fit in shared memory
  const size_t tc_smem = reduce_tc_smem(D, p.bs, R).total;
  if (R % 16 == 0 && p.bs % 16 == 0 && tc_smem <= kMaxSmem) {
    cudaError_t e = cudaFuncSetAttribute(bwd_reduce_tc_kernel<D, kBf16Rec>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(tc_smem));
    if (e != cudaSuccess) return e;
    bwd_reduce_tc_kernel<D, kBf16Rec><<<dim3(p.A, p.Hkv), kMergeThreads, tc_smem, s>>>(
        p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, dest);
    return cudaGetLastError();
  }
  const size_t staged = reduce_smem(D, p.bs, R, true).total;
  const int stage_rows = staged <= size_t(110) * 1024 ? 1 : 0;   // small enough for two CTAs per SM
  const size_t smem = reduce_smem(D, p.bs, R, stage_rows != 0).total;
  cudaError_t e = cudaFuncSetAttribute(bwd_reduce_kernel<D, kBf16Rec>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  bwd_reduce_kernel<D, kBf16Rec><<<dim3(p.A, p.Hkv), kMergeThreads, smem, s>>>(
      p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, stage_rows, dest);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                         float scale, const void* part_o, const float* part_m, const float* part_l,
                         void* o, int o_bf16, float* lse, cudaStream_t s, const MergeDest& dest) {
  if (p.partial_bf16) {
    if (p.d == 64) return merge_d<64, true>(p, q, kb, vb, scale, part_o, part_m, part_l, o, o_bf16, lse, s, dest);
    return merge_d<128, true>(p, q, kb, vb, scale, part_o, part_m, part_l, o, o_bf16, lse, s, dest);
  }
  if (p.d == 64) return merge_d<64, false>(p, q, kb, vb, scale, part_o, part_m, part_l, o, o_bf16, lse, s, dest);
  return merge_d<128, false>(p, q, kb, vb, scale, part_o, part_m, part_l, o, o_bf16, lse, s, dest);
}

cudaError_t launch_bwd_delta(const DevPlan& p, const void* o, int o_bf16, const uint16_t* dout,
                             float* delta, cudaStream_t s) {
  const int rows = p.Nq * p.Hq;
  const int warps_per_block = kMergeThreads / 32;
  int blocks = (rows + warps_per_block - 1) / warps_per_block;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  if (p.d == 64)
    delta_kernel<64><<<blocks, kMergeThreads, 0, s>>>(rows, o, o_bf16, dout, delta);
  else
    delta_kernel<128><<<blocks, kMergeThreads, 0, s>>>(rows, o, o_bf16, dout, delta);
  return cudaGetLastError();
}

cudaError_t launch_bwd_reduce(const DevPlan& p, const uint16_t* q, const uint16_t* kb,
                              const uint16_t* vb, const uint16_t* dout, const float* lse,
                              const float* delta, const void* dq_part, float scale, float* dq,
                              float* dkb, float* dvb, cudaStream_t s, const MergeDest& dest) {
  if (p.partial_bf16) {
    if (p.d == 64) return reduce_d<64, true>(p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, s, dest);
    return reduce_d<128, true>(p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, s, dest);
  }
  if (p.d == 64) return reduce_d<64, false>(p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, s, dest);
  return reduce_d<128, false>(p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, s, dest);
}

}  // namespace splitkv
