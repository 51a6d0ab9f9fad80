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
// merge: grid (A, Hkv); smem kb/vb rows of the block (bf16), staged entry ids
// ---------------------------------------------------------------------------
template <int D, bool kBf16Rec>
__global__ void __launch_bounds__(kMergeThreads, 2)
    merge_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ kb,
                 const uint16_t* __restrict__ vb, float scale_log2, const void* __restrict__ part_o,
                 const float* __restrict__ part_m, const float* __restrict__ part_l, void* __restrict__ o,
                 int o_bf16, float* __restrict__ lse, const MergeDest dest) {
  constexpr int NG = D / 16;
  using RecT = Rec<kBf16Rec>;
  constexpr int EG = 64 / (NG * RecT::RW);   // entries whose records are in flight together
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw);   // [bs][D]
  uint16_t* sVb = sKb + p.bs * D;
  int* sE = reinterpret_cast<int*>(sVb + p.bs * D);        // [kEStage]
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, u = tid & 3;
  const bool bterm = p.block_term && b >= p.bt_lo && b < p.bt_hi;   // in-block term of this block here
  for (int idx = tid; bterm && idx < p.bs * (D / 8); idx += blockDim.x) {
    const int t = idx / (D / 8), ch = idx % (D / 8);
    const size_t src = (size_t(b * p.bs + t) * p.Hkv + g) * D + ch * 8;
    *reinterpret_cast<uint4*>(sKb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(kb + src);
    *reinterpret_cast<uint4*>(sVb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(vb + src);
  }
  const int e0 = p.block_entry_ptr[b], n = p.block_entry_ptr[b + 1] - e0;
  const int R = p.G * p.bs;
  const int n_block_keys = bterm ? p.bs : 0;   // none when they are context keys, or on another rank
  // output rows: the plan's own outputs, or the owner's receive buffer (see MergeDest);
  // row_base = this block's first row in the buffer written to
  void* o_out = o;
  float* lse_out = lse;
  int out_bf16 = o_bf16;
  size_t row_base = size_t(b) * p.bs;
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
    const size_t qrow = size_t(b * p.bs + tt) * p.Hq + head;
    stage_entries(sE, p.block_entries + e0, 0, min(n, kEStage));
    // in-block term: online softmax over the bs block keys (base 2), unnormalised
    float acc[NG][4];
    float M = -INFINITY, L = 0.f;
    {
      float qv[NG][4];
      load_bf16_quad<NG>(q + qrow * D, u, qv);
#pragma unroll
      for (int k = 0; k < NG; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[k][i] = 0.f;
      for (int key = 0; key < n_block_keys; ++key) {
        float kv[NG][4];
        load_bf16_quad<NG>(sKb + key * D, u, kv);
        float dot = 0.f;
#pragma unroll
        for (int k = 0; k < NG; ++k)
#pragma unroll
          for (int i = 0; i < 4; ++i) dot = fmaf(qv[k][i], kv[k][i], dot);
        const float sc = quad_sum(dot) * scale_log2;
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
            const size_t rec = size_t(sE[i0 + v] * p.bs + tt) * p.Hq + head;
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
// dq reduce + in-block backward: grid (A, Hkv)
// smem: kb, vb [bs][D] bf16; P, dS [rows][bs] fp32 (rows = G*bs, ordered
// (token, head)); q, dout [rows][D] bf16 when stage_rows; entry ids
// ---------------------------------------------------------------------------
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
  constexpr int DPL = D / 32;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int bs = p.bs;
  const int R = p.G * bs;
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sVb = sKb + bs * D;
  float* sP = reinterpret_cast<float*>(sVb + bs * D);    // [rows][bs]
  float* sdS = sP + R * bs;                               // [rows][bs]
  int* sE = reinterpret_cast<int*>(sdS + R * bs);         // [kEStage]
  uint16_t* sQr = reinterpret_cast<uint16_t*>(sE + kEStage);   // [rows][D] when stage_rows
  uint16_t* sDr = sQr + R * D;
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, u = tid & 3, warp = tid >> 5, lane = tid & 31;
  const int nwarps = blockDim.x >> 5;
  const bool bterm = p.block_term && b >= p.bt_lo && b < p.bt_hi;   // in-block term of this block here
  for (int idx = tid; bterm && idx < bs * (D / 8); idx += blockDim.x) {
    const int t = idx / (D / 8), ch = idx % (D / 8);
    const size_t src = (size_t(b * bs + t) * p.Hkv + g) * D + ch * 8;
    *reinterpret_cast<uint4*>(sKb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(kb + src);
    *reinterpret_cast<uint4*>(sVb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(vb + src);
  }
  const int n_block_keys = bterm ? bs : 0;   // none when they are context keys, or on another rank
  // dq rows: the plan's own dq, or the owner's receive buffer (see MergeDest; dest.o)
  float* dq_out = dq;
  size_t dq_base = size_t(b) * bs;
  bool dq_ok = true;
  if (dest.o != nullptr) dq_out = dest.o[dest_of_block(p, dest, b, dq_base, dq_ok)];
  const float scale_log2 = scale * kLog2e;
  const int e0 = p.block_entry_ptr[b], n = p.block_entry_ptr[b + 1] - e0;
  // phase 1, a quad per row: P, dS of the in-block keys; dq = in-block dq + sum of partials
  for (int r0 = 0; r0 < R; r0 += kRowsPerPass) {
    const int r = min(r0 + (tid >> 2), R - 1);          // rows past R compute, never store
    const bool active = r0 + (tid >> 2) < R;
    const int tt = r / p.G, hh = r - tt * p.G;
    const int head = g * p.G + hh;
    const size_t qrow = size_t(b * bs + tt) * p.Hq + head;
    stage_entries(sE, p.block_entries + e0, 0, min(n, kEStage));
    float acc[NG][4];
    {
      float qv[NG][4], dov[NG][4];
      load_bf16_quad<NG>(q + qrow * D, u, qv);
      load_bf16_quad<NG>(dout + qrow * D, u, dov);
      const float l2 = lse[qrow] * kLog2e;
      const float dl = delta[qrow];
#pragma unroll
      for (int k = 0; k < NG; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[k][i] = 0.f;
      for (int key = 0; key < n_block_keys; ++key) {
        float sd = 0.f, dp = 0.f;
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          float kv[1][4], vv[1][4];
          load_bf16_quad<1>(sKb + key * D + 16 * k, u, kv);
          load_bf16_quad<1>(sVb + key * D + 16 * k, u, vv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            sd = fmaf(qv[k][i], kv[0][i], sd);
            dp = fmaf(dov[k][i], vv[0][i], dp);
          }
        }
        sd = quad_sum(sd);
        dp = quad_sum(dp);
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
      if (stage_rows && active && bterm) {   // keep q and dout of this row for the dkb / dvb pass
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          const int off = r * D + 4 * (u + 4 * k);
          *reinterpret_cast<uint2*>(sQr + off) = *reinterpret_cast<const uint2*>(q + qrow * D + 4 * (u + 4 * k));
          *reinterpret_cast<uint2*>(sDr + off) = *reinterpret_cast<const uint2*>(dout + qrow * D + 4 * (u + 4 * k));
        }
      }
    }
    // the in-block term, then the chunk partials in ascending chunk order, EG in flight
    float4 tot[NG];
#pragma unroll
    for (int k = 0; k < NG; ++k)
      tot[k] = make_float4(scale * acc[k][0], scale * acc[k][1], scale * acc[k][2], scale * acc[k][3]);
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
  __syncthreads();
  // phase 2, one warp per block key: dkb = scale * sum_r dS[r] q_r, dvb = sum_r P[r] dout_r
  for (int key = warp; key < n_block_keys; key += nwarps) {
    float ak[DPL], av[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) ak[i] = av[i] = 0.f;
    for (int r = 0; r < R; ++r) {
      float qv[DPL], dov[DPL];
      if (stage_rows) {
        load_bf16_row<DPL>(sQr + r * D + lane * DPL, qv);
        load_bf16_row<DPL>(sDr + r * D + lane * DPL, dov);
      } else {
        const int tt = r / p.G, hh = r - tt * p.G;
        const size_t qrow = size_t(b * bs + tt) * p.Hq + g * p.G + hh;
        load_bf16_row<DPL>(q + qrow * D + lane * DPL, qv);
        load_bf16_row<DPL>(dout + qrow * D + lane * DPL, dov);
      }
      const float ds = sdS[r * bs + key], pr = sP[r * bs + key];
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        ak[i] = fmaf(ds, qv[i], ak[i]);
        av[i] = fmaf(pr, dov[i], av[i]);
      }
    }
    const size_t krow = size_t(b * bs + key) * p.Hkv + g;
    float* dk_dst = dkb + krow * D + lane * DPL;
    float* dv_dst = dvb + krow * D + lane * DPL;
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(dk_dst) = make_float4(scale * ak[0], scale * ak[1], scale * ak[2], scale * ak[3]);
      *reinterpret_cast<float4*>(dv_dst) = make_float4(av[0], av[1], av[2], av[3]);
    } else {
      *reinterpret_cast<float2*>(dk_dst) = make_float2(scale * ak[0], scale * ak[1]);
      *reinterpret_cast<float2*>(dv_dst) = make_float2(av[0], av[1]);
    }
  }
}

template <int D, bool kBf16Rec>
cudaError_t merge_d(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                    float scale, const void* po, const float* pm, const float* pl, void* o, int o_bf16,
                    float* lse, cudaStream_t s, const MergeDest& dest) {
  const size_t smem = size_t(2) * p.bs * D * sizeof(uint16_t) + kEStage * sizeof(int);
  cudaError_t e =
      cudaFuncSetAttribute(merge_kernel<D, kBf16Rec>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  merge_kernel<D, kBf16Rec><<<dim3(p.A, p.Hkv), kMergeThreads, smem, s>>>(p, q, kb, vb, scale * kLog2e, po, pm,
                                                                            pl, o, o_bf16, lse, dest);
  return cudaGetLastError();
}

template <int D, bool kBf16Rec>
cudaError_t reduce_d(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                     const uint16_t* dout, const float* lse, const float* delta, const void* dq_part,
                     float scale, float* dq, float* dkb, float* dvb, cudaStream_t s, const MergeDest& dest) {
  const size_t rows = size_t(p.G) * p.bs;
  const size_t base =
      size_t(2) * p.bs * D * sizeof(uint16_t) + 2 * rows * p.bs * sizeof(float) + kEStage * sizeof(int);
  const size_t staged = base + 2 * rows * D * sizeof(uint16_t);
  const int stage_rows = staged <= size_t(64) * 1024 ? 1 : 0;   // small enough to keep occupancy
  const size_t smem = stage_rows ? staged : base;
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
