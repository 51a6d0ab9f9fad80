// Backward of the chunk partial attention with keys/values local to their chunk:
// warp-level mma.sync kernel.
//
// News page "Split-KV speeds diffusion drafter training by keeping long-context
// data local", section "Exchange the smaller side": key/value shards stay local
// through the forward and the backward pass.  Each (chunk, KV head) item is
// owned by one persistent CTA, which therefore owns dk/dv of its chunk (summed
// over the G query heads, no atomics); dq is written per (chunk, block) entry
// as a partial that a later kernel reduces in ascending chunk order.
//
// P is recomputed from the saved log-sum-exp: P = exp(s - lse).  For every
// 64-key tile of the chunk (warp w owns keys 16w..16w+15) the CTA visits the
// 32-row sub-tiles of every query tile that meets the key tile and computes,
// keys as the MMA's M dimension:
//   S^T = K Q^T; P^T; dV += P^T dO; dP^T = V dO^T; dS^T = P^T (dP^T - Delta);
//   dK += dS^T Q; dQ_sub = dS K (through shared memory) -> the entry's partial.
// dQ partial rows are stored by the first key tile that meets their query tile
// and accumulated with fire-and-forget reductions afterwards; one thread always
// owns the same element, so the summation order is fixed.
#include <cfloat>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "splitkv_internal.h"

namespace splitkv {
namespace {

constexpr int kBN = 64;   // keys per key tile
constexpr int kBM = 32;   // query rows per sub-tile
constexpr int kThreads = 128;

template <int D>
constexpr size_t bwd_smem_bytes() {
  return size_t(2 * kBN * D + 4 * kBM * D + kBM * kBN) * sizeof(uint16_t) + 2 * 5 * kBM * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_partial_mma_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                           const uint16_t* __restrict__ v, const uint16_t* __restrict__ dout,
                           const float* __restrict__ lse, const float* __restrict__ delta, float scale,
                           float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dq_part) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(smem_raw);   // [kBN][D]
  uint16_t* sV = sK + kBN * D;                             // [kBN][D]
  uint16_t* sQ = sV + kBN * D;                             // [2][kBM][D]
  uint16_t* sdO = sQ + 2 * kBM * D;                        // [2][kBM][D]
  uint16_t* sdS = sdO + 2 * kBM * D;                       // [kBM][kBN], swizzled as D = 64
  float* sLse2 = reinterpret_cast<float*>(sdS + kBM * kBN);  // [2][kBM]
  float* sDelta = sLse2 + 2 * kBM;
  int* sLo = reinterpret_cast<int*>(sDelta + 2 * kBM);
  int* sHi = sLo + 2 * kBM;
  int* sRec = sHi + 2 * kBM;

  const int w = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) p.timers[(p.W + w) * 2 + 0] = global_timer_ns();
  constexpr int CH = D / 8;
  const size_t kv_row = size_t(p.Hkv) * D;
  const float scale_log2 = scale * kLog2e;
  const int rows_per_slot = p.G * p.bs;

  // chunks that no block reads: dk = dv = 0 for every KV head
  for (int z = w; z < p.num_zero_chunks; z += p.Wb) {
    const int c = p.zero_chunks[z];
    const size_t first = size_t(c) * p.C * kv_row;
    const size_t last = size_t(min(c * p.C + p.C, p.N)) * kv_row;
    for (size_t i = first + size_t(tid) * 4; i < last; i += size_t(kThreads) * 4) {
      *reinterpret_cast<float4*>(dk + i) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(dv + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  for (int it = p.bwd_worker_ptr[w]; it < p.bwd_worker_ptr[w + 1]; ++it) {
    const int4 item = p.bwd_items[it];  // chunk, kv head, t0, t1
    const int c = item.x, g = item.y;
    const int c0 = c * p.C, c1 = min(c0 + p.C, p.N);
    const uint16_t* kg = k + size_t(g) * D;
    const uint16_t* vg = v + size_t(g) * D;

    // does query tile t meet key tile [kt0, kt0 + kBN)?
    auto meets = [&](int t, int kt0) {
      const int4 tl = p.tiles[t];
      return tl.z < kt0 + kBN && tl.w > kt0;
    };
    // next (tile, sub) unit at or after (t, sub) that meets the key tile; t == item.w when done
    auto advance = [&](int& t, int& sub, int kt0) {
      while (t < item.w) {
        if (sub < kTileRows / kBM && meets(t, kt0)) {
          const int4 tl = p.tiles[t];
          if (sub * kBM < (tl.y - tl.x) * rows_per_slot) return;
        }
        ++t;
        sub = 0;
      }
    };
    auto load_unit = [&](int t, int sub, int buf) {
      const int4 tl = p.tiles[t];
      const int nslots = tl.y - tl.x;
      uint16_t* dq_s = sQ + buf * kBM * D;
      uint16_t* do_s = sdO + buf * kBM * D;
      for (int idx = tid; idx < kBM * CH; idx += kThreads) {
        const int r = idx / CH, ch = idx % CH;
        const int R = sub * kBM + r;
        const int slot = R / rows_per_slot;
        const bool valid = slot < nslots;
        size_t off = 0;
        if (valid) {
          const int bb = p.entries[tl.x + slot].x;
          const int hh = (R % rows_per_slot) / p.bs, tt = R % p.bs;
          off = (size_t(bb * p.bs + tt) * p.Hq + g * p.G + hh) * D + ch * 8;
        }
        cp_async16(dq_s + swz<D>(r, ch), q + off, valid);
        cp_async16(do_s + swz<D>(r, ch), dout + off, valid);
      }
      if (tid < kBM) {
        const int r = tid;
        const int R = sub * kBM + r;
        const int slot = R / rows_per_slot;
        float l2 = INFINITY, dl = 0.f;
        int lo = 0, hi = 0, rec = -1;
        if (slot < nslots) {
          const int e = tl.x + slot;
          const int4 ent = p.entries[e];
          const int hh = (R % rows_per_slot) / p.bs, tt = R % p.bs;
          const size_t qrow = size_t(ent.x * p.bs + tt) * p.Hq + g * p.G + hh;
          const float L = lse[qrow];
          l2 = (L == -INFINITY) ? INFINITY : L * kLog2e;
          dl = delta[qrow];
          lo = ent.y;
          hi = ent.z;
          rec = (e * p.bs + tt) * p.Hq + g * p.G + hh;
        }
        sLse2[buf * kBM + r] = l2;
        sDelta[buf * kBM + r] = dl;
        sLo[buf * kBM + r] = lo;
        sHi[buf * kBM + r] = hi;
        sRec[buf * kBM + r] = rec;
      }
    };

    for (int kt0 = c0; kt0 < c1; kt0 += kBN) {
      // K, V tile of the chunk (keys beyond the chunk read as zero)
      for (int idx = tid; idx < kBN * CH; idx += kThreads) {
        const int r = idx / CH, ch = idx % CH;
        const int key = kt0 + r;
        const bool valid = key < c1;
        const size_t off = size_t(valid ? key : c0) * kv_row + ch * 8;
        cp_async16(sK + swz<D>(r, ch), kg + off, valid);
        cp_async16(sV + swz<D>(r, ch), vg + off, valid);
      }
      int t = item.z, sub = 0;
      advance(t, sub, kt0);
      if (t < item.w) load_unit(t, sub, 0);
      cp_async_commit();

      float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
      for (int i = 0; i < D / 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dka[i][j] = dva[i][j] = 0.f;

      const int key_a = kt0 + warp * 16 + (lane >> 2), key_b = key_a + 8;
      int buf = 0;
      while (t < item.w) {
        // prefetch the next unit into the other buffer
        int tn = t, sn = sub + 1;
        advance(tn, sn, kt0);
        if (tn < item.w) load_unit(tn, sn, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        const uint16_t* bq = sQ + buf * kBM * D;
        const uint16_t* bdo = sdO + buf * kBM * D;
        const float* lse2 = sLse2 + buf * kBM;
        const float* dlt = sDelta + buf * kBM;
        const int* rlo = sLo + buf * kBM;
        const int* rhi = sHi + buf * kBM;

        // S^T = K_w Q^T and dP^T = V_w dO^T (16 keys x 32 rows each)
        float st[kBM / 8][4], dpt[kBM / 8][4];
#pragma unroll
        for (int i = 0; i < kBM / 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) st[i][j] = dpt[i][j] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t ak[4], av[4];
          const int ar = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
          const int ach = 2 * kk + (lane >> 4);
          ldsm_x4(ak[0], ak[1], ak[2], ak[3], sK + swz<D>(ar, ach));
          ldsm_x4(av[0], av[1], av[2], av[3], sV + swz<D>(ar, ach));
#pragma unroll
          for (int np = 0; np < kBM / 16; ++np) {
            const int n = np * 16 + (lane & 7) + 8 * (lane >> 4);
            const int ch = 2 * kk + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(b0, b1, b2, b3, bq + swz<D>(n, ch));
            mma_bf16_16816(st[2 * np], ak, b0, b1);
            mma_bf16_16816(st[2 * np + 1], ak, b2, b3);
            ldsm_x4(b0, b1, b2, b3, bdo + swz<D>(n, ch));
            mma_bf16_16816(dpt[2 * np], av, b0, b1);
            mma_bf16_16816(dpt[2 * np + 1], av, b2, b3);
          }
        }
        // P^T and dS^T (thread: keys key_a/key_b, rows nb*8 + 2*(lane&3) + e)
#pragma unroll
        for (int nb = 0; nb < kBM / 8; ++nb) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = nb * 8 + 2 * (lane & 3) + e;
            const int lo = rlo[r], hi = rhi[r];
            const float l2 = lse2[r], dl = dlt[r];
            const float pa = (key_a >= lo && key_a < hi) ? fast_exp2(st[nb][e] * scale_log2 - l2) : 0.f;
            const float pb = (key_b >= lo && key_b < hi) ? fast_exp2(st[nb][2 + e] * scale_log2 - l2) : 0.f;
            st[nb][e] = pa;
            st[nb][2 + e] = pb;
            dpt[nb][e] = pa * (dpt[nb][e] - dl);
            dpt[nb][2 + e] = pb * (dpt[nb][2 + e] - dl);
          }
        }
        // dV += P^T dO, dK += dS^T Q (k-steps over the 32 rows)
#pragma unroll
        for (int ks = 0; ks < kBM / 16; ++ks) {
          uint32_t pa[4], sa[4];
          pa[0] = pack_bf16(st[2 * ks][0], st[2 * ks][1]);
          pa[1] = pack_bf16(st[2 * ks][2], st[2 * ks][3]);
          pa[2] = pack_bf16(st[2 * ks + 1][0], st[2 * ks + 1][1]);
          pa[3] = pack_bf16(st[2 * ks + 1][2], st[2 * ks + 1][3]);
          sa[0] = pack_bf16(dpt[2 * ks][0], dpt[2 * ks][1]);
          sa[1] = pack_bf16(dpt[2 * ks][2], dpt[2 * ks][3]);
          sa[2] = pack_bf16(dpt[2 * ks + 1][0], dpt[2 * ks + 1][1]);
          sa[3] = pack_bf16(dpt[2 * ks + 1][2], dpt[2 * ks + 1][3]);
#pragma unroll
          for (int dp = 0; dp < D / 16; ++dp) {
            const int kr = ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ch = 2 * dp + (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(b0, b1, b2, b3, bdo + swz<D>(kr, ch));
            mma_bf16_16816(dva[2 * dp], pa, b0, b1);
            mma_bf16_16816(dva[2 * dp + 1], pa, b2, b3);
            ldsm_x4_t(b0, b1, b2, b3, bq + swz<D>(kr, ch));
            mma_bf16_16816(dka[2 * dp], sa, b0, b1);
            mma_bf16_16816(dka[2 * dp + 1], sa, b2, b3);
          }
        }
        // dS (bf16) to shared memory as [row][key] for the dQ product
        {
          const int kl_a = warp * 16 + (lane >> 2), kl_b = kl_a + 8;
#pragma unroll
          for (int nb = 0; nb < kBM / 8; ++nb) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int r = nb * 8 + 2 * (lane & 3) + e;
              const __nv_bfloat16 va = __float2bfloat16_rn(dpt[nb][e]);
              const __nv_bfloat16 vb = __float2bfloat16_rn(dpt[nb][2 + e]);
              sdS[swz<kBN>(r, kl_a >> 3) + (kl_a & 7)] = *reinterpret_cast<const uint16_t*>(&va);
              sdS[swz<kBN>(r, kl_b >> 3) + (kl_b & 7)] = *reinterpret_cast<const uint16_t*>(&vb);
            }
          }
        }
        __syncthreads();
        // dQ_sub (32 rows x D) = dS (32 x 64) K (64 x D); warp: rows 16*(w&1), d half (w>>1)
        {
          float dqa[D / 16][4];
#pragma unroll
          for (int i = 0; i < D / 16; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;
          const int rbase = 16 * (warp & 1);
          const int cbase = (warp >> 1) * (D / 16);   // chunk offset of this d half
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks) {
            uint32_t a[4];
            const int ar = rbase + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ach = 2 * ks + (lane >> 4);
            ldsm_x4(a[0], a[1], a[2], a[3], sdS + swz<kBN>(ar, ach));
#pragma unroll
            for (int dp = 0; dp < D / 32; ++dp) {
              const int kr = ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
              const int ch = cbase + 2 * dp + (lane >> 4);
              uint32_t b0, b1, b2, b3;
              ldsm_x4_t(b0, b1, b2, b3, sK + swz<D>(kr, ch));
              mma_bf16_16816(dqa[2 * dp], a, b0, b1);
              mma_bf16_16816(dqa[2 * dp + 1], a, b2, b3);
            }
          }
          const int4 tl = p.tiles[t];
          const bool first = tl.z >= kt0 && tl.z < kt0 + kBN;   // first key tile meeting this query tile
          const int ra = rbase + (lane >> 2), rb = ra + 8;
          const int rec_a = sRec[buf * kBM + ra], rec_b = sRec[buf * kBM + rb];
          const int col0 = (warp >> 1) * (D / 2) + 2 * (lane & 3);
#pragma unroll
          for (int nb = 0; nb < D / 16; ++nb) {
            const int col = col0 + nb * 8;
            if (rec_a >= 0) {
              float* dst = dq_part + size_t(rec_a) * D + col;
              if (first) {
                *reinterpret_cast<float2*>(dst) = make_float2(scale * dqa[nb][0], scale * dqa[nb][1]);
              } else {
                atomicAdd(dst, scale * dqa[nb][0]);
                atomicAdd(dst + 1, scale * dqa[nb][1]);
              }
            }
            if (rec_b >= 0) {
              float* dst = dq_part + size_t(rec_b) * D + col;
              if (first) {
                *reinterpret_cast<float2*>(dst) = make_float2(scale * dqa[nb][2], scale * dqa[nb][3]);
              } else {
                atomicAdd(dst, scale * dqa[nb][2]);
                atomicAdd(dst + 1, scale * dqa[nb][3]);
              }
            }
          }
        }
        __syncthreads();   // buffers and sdS are reused by the next unit
        t = tn;
        sub = sn;
        buf ^= 1;
      }
      cp_async_wait<0>();
      __syncthreads();
      // dk (scaled), dv of the warp's 16 keys
      const int col0 = 2 * (lane & 3);
#pragma unroll
      for (int nb = 0; nb < D / 8; ++nb) {
        const int col = nb * 8 + col0;
        if (key_a < c1) {
          const size_t off = (size_t(key_a) * p.Hkv + g) * D + col;
          *reinterpret_cast<float2*>(dk + off) = make_float2(scale * dka[nb][0], scale * dka[nb][1]);
          *reinterpret_cast<float2*>(dv + off) = make_float2(dva[nb][0], dva[nb][1]);
        }
        if (key_b < c1) {
          const size_t off = (size_t(key_b) * p.Hkv + g) * D + col;
          *reinterpret_cast<float2*>(dk + off) = make_float2(scale * dka[nb][2], scale * dka[nb][3]);
          *reinterpret_cast<float2*>(dv + off) = make_float2(dva[nb][2], dva[nb][3]);
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) p.timers[(p.W + w) * 2 + 1] = global_timer_ns();
}

template <int D>
cudaError_t launch_bwd_d(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const uint16_t* dout, const float* lse, const float* delta, float scale,
                         float* dk, float* dv, float* dq_part, cudaStream_t s) {
  const size_t smem = bwd_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(bwd_partial_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  bwd_partial_mma_kernel<D><<<p.Wb, kThreads, smem, s>>>(p, q, k, v, dout, lse, delta, scale, dk, dv, dq_part);
  return cudaGetLastError();
}

}  // namespace

bool bwd_sm100_supported(const DevPlan& p);
cudaError_t launch_bwd_partial_sm100(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     const uint16_t* dout, const float* lse, const float* delta, float scale,
                                     float* dk, float* dv, void* dq_part, cudaStream_t s, int which);

// The tcgen05 kernels serve head_dim 128 with G * bs a multiple of 8; every
// other shape runs the mma.sync kernel.  SPLITKV_BWD_KERNEL=mma selects the
// mma.sync kernel for every shape (for comparisons).
cudaError_t launch_bwd_partial(const DevPlan& p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const uint16_t* dout, const float* lse,
                               const float* delta, float scale, float* dk, float* dv,
                               void* dq_part, cudaStream_t s, int which) {
  static const bool force_mma = [] {
    const char* e = std::getenv("SPLITKV_BWD_KERNEL");
    return e != nullptr && std::strcmp(e, "mma") == 0;
  }();
  if (!force_mma && bwd_sm100_supported(p))
    return launch_bwd_partial_sm100(p, q, k, v, dout, lse, delta, scale, dk, dv, dq_part, s, which);
  if (p.partial_bf16 || p.dynamic) return cudaErrorNotSupported;   // the entry points check this first
  if (which == 2) return cudaSuccess;   // the single mma.sync kernel ran in the dK/dV part
  float* dqp = static_cast<float*>(dq_part);
  if (p.d == 64) return launch_bwd_d<64>(p, q, k, v, dout, lse, delta, scale, dk, dv, dqp, s);
  return launch_bwd_d<128>(p, q, k, v, dout, lse, delta, scale, dk, dv, dqp, s);
}

}  // namespace splitkv
