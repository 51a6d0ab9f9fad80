// HBM-bound kernels around the partial-attention kernels:
//   merge_kernel        exact log-sum-exp combine of a block's chunk records plus
//                       its in-block term -> o, lse
//   delta_kernel        Delta_i = dout_i . o_i (backward preamble)
//   bwd_reduce_kernel   dq = sum of chunk dq partials (ascending chunk) + the
//                       in-block term's dq; dkb, dvb of the in-block term
//
// News page "Split-KV speeds diffusion drafter training by keeping long-context
// data local", section "Exchange the smaller side" (partials combined exactly
// with their normalisation statistics) and section "Why short queries change
// the problem" (every block also attends to all tokens inside itself; those
// bs keys are the draft block's own kb/vb rows).
//
// One CTA per (block b, KV head g) handles the G*bs query rows (G heads x bs
// tokens) that read the same bs block keys; one warp per row, each lane owning
// D/32 consecutive dimensions, so every record row is a coalesced 256/512-byte
// read.  All loops run in a fixed order, so results are deterministic.
#include <cfloat>

#include "common.cuh"
#include "splitkv_internal.h"

namespace splitkv {
namespace {

constexpr int kMergeThreads = 256;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

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
// merge: grid (A, Hkv), smem kb/vb rows of the block (bf16)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    merge_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ kb,
                 const uint16_t* __restrict__ vb, float scale_log2, const float* __restrict__ part_o,
                 const float* __restrict__ part_m, const float* __restrict__ part_l, void* __restrict__ o,
                 int o_bf16, float* __restrict__ lse) {
  constexpr int DPL = D / 32;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw);   // [bs][D]
  uint16_t* sVb = sKb + p.bs * D;
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = blockDim.x >> 5;
  // stage the block's own keys/values of KV head g
  for (int idx = tid; idx < p.bs * (D / 8); idx += blockDim.x) {
    const int t = idx / (D / 8), ch = idx % (D / 8);
    const size_t src = (size_t(b * p.bs + t) * p.Hkv + g) * D + ch * 8;
    *reinterpret_cast<uint4*>(sKb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(kb + src);
    *reinterpret_cast<uint4*>(sVb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(vb + src);
  }
  __syncthreads();
  const int e0 = p.block_entry_ptr[b], e1 = p.block_entry_ptr[b + 1];
  const int rows = p.G * p.bs;
  for (int r = warp; r < rows; r += nwarps) {
    const int hh = r / p.bs, tt = r % p.bs;
    const int head = g * p.G + hh;
    const size_t qrow = size_t(b * p.bs + tt) * p.Hq + head;
    float qv[DPL];
    load_bf16_row<DPL>(q + qrow * D + lane * DPL, qv);
    // in-block term: online softmax over the bs block keys (base 2)
    float mb = -INFINITY, lb = 0.f, ob[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) ob[i] = 0.f;
    for (int key = 0; key < p.bs; ++key) {
      float kv[DPL], vv[DPL];
      load_bf16_row<DPL>(sKb + key * D + lane * DPL, kv);
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) dot = fmaf(qv[i], kv[i], dot);
      const float s = warp_sum(dot) * scale_log2;
      const float mn = fmaxf(mb, s);
      const float corr = fast_exp2(mb - mn);
      const float pr = fast_exp2(s - mn);
      lb = lb * corr + pr;
      load_bf16_row<DPL>(sVb + key * D + lane * DPL, vv);
#pragma unroll
      for (int i = 0; i < DPL; ++i) ob[i] = ob[i] * corr + pr * vv[i];
      mb = mn;
    }
    // the chunk records of this row: one entry per lane, 32 at a time
    const int n = e1 - e0;
    float Mc = -INFINITY;
    for (int base = 0; base < n; base += 32) {
      float m2 = -INFINITY;
      if (base + lane < n) {
        const int rec = (p.block_entries[e0 + base + lane] * p.bs + tt) * p.Hq + head;
        if (part_l[rec] > 0.f) m2 = part_m[rec] * kLog2e;
      }
      Mc = fmaxf(Mc, warp_max(m2));
    }
    const float M = fmaxf(mb, Mc);
    const float wb = fast_exp2(mb - M);   // ob is unnormalised: weight exp2(mb - M)
    float L = lb * wb;
    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = ob[i] * wb;
    // weighted sum of the normalised chunk outputs in ascending chunk order, 8 rows in flight
    for (int base = 0; base < n; base += 32) {
      float wl = 0.f;
      int recl = 0;
      if (base + lane < n) {
        recl = (p.block_entries[e0 + base + lane] * p.bs + tt) * p.Hq + head;
        const float lx = part_l[recl];
        wl = lx > 0.f ? lx * fast_exp2(part_m[recl] * kLog2e - M) : 0.f;
      }
      L += warp_sum(wl);
      const int cnt = min(32, n - base);
      for (int j0 = 0; j0 < cnt; j0 += 8) {
        float w8[8];
        float ov[8][DPL];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u;
          const float wj = __shfl_sync(0xffffffffu, wl, j & 31);
          const int rj = __shfl_sync(0xffffffffu, recl, j & 31);
          w8[u] = j < cnt ? wj : 0.f;
          if (j < cnt) {
            load_f32_row<DPL>(part_o + size_t(rj) * D + lane * DPL, ov[u]);
          } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) ov[u][i] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w8[u], ov[u][i], acc[i]);
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if (o_bf16) {
      uint16_t* dst = static_cast<uint16_t*>(o) + qrow * D + lane * DPL;
      if constexpr (DPL == 4) {
        uint2 u;
        u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
        u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(dst) = u;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
      }
    } else {
      float* dst = static_cast<float*>(o) + qrow * D + lane * DPL;
      if constexpr (DPL == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      } else {
        *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
      }
    }
    if (lane == 0) lse[qrow] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
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
// smem: kb, vb [bs][D] bf16; P, dS [rows][bs] fp32 (rows = G*bs)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    bwd_reduce_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ kb,
                      const uint16_t* __restrict__ vb, const uint16_t* __restrict__ dout,
                      const float* __restrict__ lse, const float* __restrict__ delta,
                      const float* __restrict__ dq_part, float scale, float* __restrict__ dq,
                      float* __restrict__ dkb, float* __restrict__ dvb, int stage_rows) {
  constexpr int DPL = D / 32;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int bs = p.bs;
  const int rows = p.G * bs;
  uint16_t* sKb = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sVb = sKb + bs * D;
  float* sP = reinterpret_cast<float*>(sVb + bs * D);    // [rows][bs]
  float* sdS = sP + rows * bs;                            // [rows][bs]
  uint16_t* sQr = reinterpret_cast<uint16_t*>(sdS + rows * bs);   // [rows][D] when stage_rows
  uint16_t* sDr = sQr + rows * D;
  const int b = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = blockDim.x >> 5;
  for (int idx = tid; idx < bs * (D / 8); idx += blockDim.x) {
    const int t = idx / (D / 8), ch = idx % (D / 8);
    const size_t src = (size_t(b * bs + t) * p.Hkv + g) * D + ch * 8;
    *reinterpret_cast<uint4*>(sKb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(kb + src);
    *reinterpret_cast<uint4*>(sVb + t * D + ch * 8) = *reinterpret_cast<const uint4*>(vb + src);
  }
  __syncthreads();
  const float scale_log2 = scale * kLog2e;
  const int e0 = p.block_entry_ptr[b], e1 = p.block_entry_ptr[b + 1];
  // phase 1, one warp per row: P, dS of the in-block keys; dq = sum of partials + in-block dq
  for (int r = warp; r < rows; r += nwarps) {
    const int hh = r / bs, tt = r % bs;
    const int head = g * p.G + hh;
    const size_t qrow = size_t(b * bs + tt) * p.Hq + head;
    float qv[DPL], dov[DPL];
    load_bf16_row<DPL>(q + qrow * D + lane * DPL, qv);
    load_bf16_row<DPL>(dout + qrow * D + lane * DPL, dov);
    const float l2 = lse[qrow] * kLog2e;
    const float dl = delta[qrow];
    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
    for (int key = 0; key < bs; ++key) {
      float kv[DPL], vv[DPL];
      load_bf16_row<DPL>(sKb + key * D + lane * DPL, kv);
      load_bf16_row<DPL>(sVb + key * D + lane * DPL, vv);
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        s = fmaf(qv[i], kv[i], s);
        dp = fmaf(dov[i], vv[i], dp);
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      const float pr = (l2 == -INFINITY) ? 0.f : fast_exp2(s * scale_log2 - l2);
      const float ds = pr * (dp - dl);
      if (lane == 0) {
        sP[r * bs + key] = pr;
        sdS[r * bs + key] = ds;
      }
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(ds, kv[i], acc[i]);
    }
    // chunk partials in ascending chunk order (8 rows in flight), then the in-block term
    float tot[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) tot[i] = 0.f;
    const int n = e1 - e0;
    for (int base = 0; base < n; base += 32) {
      int recl = 0;
      if (base + lane < n) recl = (p.block_entries[e0 + base + lane] * bs + tt) * p.Hq + head;
      const int cnt = min(32, n - base);
      for (int j0 = 0; j0 < cnt; j0 += 8) {
        float pv[8][DPL];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u;
          const int rj = __shfl_sync(0xffffffffu, recl, j & 31);
          if (j < cnt) {
            load_f32_row<DPL>(dq_part + size_t(rj) * D + lane * DPL, pv[u]);
          } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) pv[u][i] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int i = 0; i < DPL; ++i) tot[i] += pv[u][i];
      }
    }
    if (stage_rows) {   // keep q and dout of this row for the dkb / dvb pass
      uint16_t* sq = sQr + r * D + lane * DPL;
      uint16_t* sd = sDr + r * D + lane * DPL;
      if constexpr (DPL == 4) {
        *reinterpret_cast<uint2*>(sq) = *reinterpret_cast<const uint2*>(q + qrow * D + lane * DPL);
        *reinterpret_cast<uint2*>(sd) = *reinterpret_cast<const uint2*>(dout + qrow * D + lane * DPL);
      } else {
        *reinterpret_cast<uint32_t*>(sq) = *reinterpret_cast<const uint32_t*>(q + qrow * D + lane * DPL);
        *reinterpret_cast<uint32_t*>(sd) = *reinterpret_cast<const uint32_t*>(dout + qrow * D + lane * DPL);
      }
    }
    float* dst = dq + qrow * D + lane * DPL;
#pragma unroll
    for (int i = 0; i < DPL; ++i) tot[i] += scale * acc[i];
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(dst) = make_float4(tot[0], tot[1], tot[2], tot[3]);
    } else {
      *reinterpret_cast<float2*>(dst) = make_float2(tot[0], tot[1]);
    }
  }
  __syncthreads();
  // phase 2, one warp per block key: dkb = scale * sum_r dS[r] q_r, dvb = sum_r P[r] dout_r
  for (int key = warp; key < bs; key += nwarps) {
    float ak[DPL], av[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) ak[i] = av[i] = 0.f;
    for (int r = 0; r < rows; ++r) {
      float qv[DPL], dov[DPL];
      if (stage_rows) {
        load_bf16_row<DPL>(sQr + r * D + lane * DPL, qv);
        load_bf16_row<DPL>(sDr + r * D + lane * DPL, dov);
      } else {
        const int hh = r / bs, tt = r % bs;
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

template <int D>
cudaError_t merge_d(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                    float scale, const float* po, const float* pm, const float* pl, void* o, int o_bf16,
                    float* lse, cudaStream_t s) {
  const size_t smem = size_t(2) * p.bs * D * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(merge_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  merge_kernel<D><<<dim3(p.A, p.Hkv), kMergeThreads, smem, s>>>(p, q, kb, vb, scale * kLog2e, po, pm, pl, o,
                                                                  o_bf16, lse);
  return cudaGetLastError();
}

template <int D>
cudaError_t reduce_d(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                     const uint16_t* dout, const float* lse, const float* delta, const float* dq_part,
                     float scale, float* dq, float* dkb, float* dvb, cudaStream_t s) {
  const size_t rows = size_t(p.G) * p.bs;
  const size_t base = size_t(2) * p.bs * D * sizeof(uint16_t) + 2 * rows * p.bs * sizeof(float);
  const size_t staged = base + 2 * rows * D * sizeof(uint16_t);
  const int stage_rows = staged <= size_t(64) * 1024 ? 1 : 0;   // small enough to keep occupancy
  const size_t smem = stage_rows ? staged : base;
  cudaError_t e =
      cudaFuncSetAttribute(bwd_reduce_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  bwd_reduce_kernel<D><<<dim3(p.A, p.Hkv), kMergeThreads, smem, s>>>(p, q, kb, vb, dout, lse, delta, dq_part,
                                                                       scale, dq, dkb, dvb, stage_rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const DevPlan& p, const uint16_t* q, const uint16_t* kb, const uint16_t* vb,
                         float scale, const float* part_o, const float* part_m, const float* part_l,
                         void* o, int o_bf16, float* lse, cudaStream_t s) {
  if (p.d == 64) return merge_d<64>(p, q, kb, vb, scale, part_o, part_m, part_l, o, o_bf16, lse, s);
  return merge_d<128>(p, q, kb, vb, scale, part_o, part_m, part_l, o, o_bf16, lse, s);
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
                              const float* delta, const float* dq_part, float scale, float* dq,
                              float* dkb, float* dvb, cudaStream_t s) {
  if (p.d == 64) return reduce_d<64>(p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, s);
  return reduce_d<128>(p, q, kb, vb, dout, lse, delta, dq_part, scale, dq, dkb, dvb, s);
}

}  // namespace splitkv
