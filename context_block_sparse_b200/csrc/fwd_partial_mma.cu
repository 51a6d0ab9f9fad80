// Partial attention of every (chunk, block) entry: warp-level mma.sync kernel.
//
// News page "Split-KV speeds diffusion drafter training by keeping long-context
// data local", section "Exchange the smaller side": each key/value shard
// evaluates every query against its own keys and emits partial results with
// their normalisation statistics.  Here a shard is a KV chunk and a worker is a
// persistent CTA that walks the items its LPT schedule gave it.
//
// Per 128-row query tile (128 / (G*bs) blocks x G heads of one KV head x bs
// tokens, rows ordered (block slot, head, token)), the CTA streams the tile's
// key union [klo, khi) through shared memory in 64-key tiles (cp.async, double
// buffered), computes S = Q K^T with mma.sync m16n8k16 (bf16 in, fp32
// accumulate), masks every row to its block's [lo, hi), keeps a base-2 online
// softmax per row in registers and accumulates O += P V.  Each warp owns 16 rows.
#include <cfloat>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "splitkv_internal.h"

namespace splitkv {
namespace {

constexpr int kBM = kTileRows;  // 128 query rows per tile
constexpr int kBN = 64;         // keys per key tile
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <int D>
constexpr size_t fwd_smem_bytes() {
  return size_t(kBM + 4 * kBN) * D * sizeof(uint16_t) + 3 * kBM * sizeof(int);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_partial_mma_kernel(DevPlan p, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                           const uint16_t* __restrict__ v, float scale_log2, float* __restrict__ part_o,
                           float* __restrict__ part_m, float* __restrict__ part_l) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sK = sQ + kBM * D;        // [2][kBN][D]
  uint16_t* sV = sK + 2 * kBN * D;    // [2][kBN][D]
  int* sLo = reinterpret_cast<int*>(sV + 2 * kBN * D);
  int* sHi = sLo + kBM;
  int* sRow = sHi + kBM;              // record row (e*bs + t)*Hq + head, or -1

  const int w = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) p.timers[w * 2 + 0] = global_timer_ns();

  const int rows_per_slot = p.G * p.bs;
  const size_t kv_row = size_t(p.Hkv) * D;   // elements between consecutive keys
  constexpr int CH = D / 8;                  // 16-byte chunks per row

  for (int it = p.fwd_worker_ptr[w]; it < p.fwd_worker_ptr[w + 1]; ++it) {
    const int4 item = p.fwd_items[it];       // chunk, kv head, t0, t1
    const int g = item.y;
    const uint16_t* kg = k + size_t(g) * D;
    const uint16_t* vg = v + size_t(g) * D;
    for (int t = item.z; t < item.w; ++t) {
      const int4 tile = p.tiles[t];          // e0, e1, klo, khi
      const int nslots = tile.y - tile.x;
      __syncthreads();                       // previous tile done with smem
      for (int r = tid; r < kBM; r += kThreads) {
        const int slot = r / rows_per_slot;
        if (slot < nslots) {
          const int e = tile.x + slot;
          const int4 ent = p.entries[e];     // block, lo, hi, chunk
          const int hh = (r % rows_per_slot) / p.bs, tt = r % p.bs;
          sRow[r] = (e * p.bs + tt) * p.Hq + g * p.G + hh;
          sLo[r] = ent.y;
          sHi[r] = ent.z;
        } else {                             // padding row: everything masked, nothing written
          sRow[r] = -1;
          sLo[r] = 0;
          sHi[r] = 0;
        }
      }
      __syncthreads();
      // Q tile (zero rows for empty slots)
      for (int idx = tid; idx < kBM * CH; idx += kThreads) {
        const int r = idx / CH, ch = idx % CH;
        const int slot = r / rows_per_slot;
        const bool valid = slot < nslots;
        const uint16_t* src = q;
        if (valid) {
          const int b = p.entries[tile.x + slot].x;
          const int hh = (r % rows_per_slot) / p.bs, tt = r % p.bs;
          src = q + (size_t(b * p.bs + tt) * p.Hq + g * p.G + hh) * D + ch * 8;
        }
        cp_async16(sQ + swz<D>(r, ch), src, valid);
      }
      const int klo = tile.z, khi = tile.w;
      const int n_kt = (khi - klo + kBN - 1) / kBN;
      auto load_kv = [&](int j, int buf) {
        uint16_t* dk = sK + buf * kBN * D;
        uint16_t* dv = sV + buf * kBN * D;
        const int kbase = klo + j * kBN;
        for (int idx = tid; idx < kBN * CH; idx += kThreads) {
          const int r = idx / CH, ch = idx % CH;
          const int key = kbase + r;
          const bool valid = key < khi;
          const size_t off = size_t(valid ? key : klo) * kv_row + ch * 8;
          cp_async16(dk + swz<D>(r, ch), kg + off, valid);
          cp_async16(dv + swz<D>(r, ch), vg + off, valid);
        }
      };
      load_kv(0, 0);
      cp_async_commit();

      // per-thread rows: ra = 16*warp + lane/4, rb = ra + 8
      const int ra = warp * 16 + (lane >> 2), rb = ra + 8;
      const int lo_a = sLo[ra], hi_a = sHi[ra], lo_b = sLo[rb], hi_b = sHi[rb];
      float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
      float o[D / 8][4];
#pragma unroll
      for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      uint32_t qa[D / 16][4];

      for (int j = 0; j < n_kt; ++j) {
        const int buf = j & 1;
        if (j + 1 < n_kt) load_kv(j + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (j == 0) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ch = 2 * kk + (lane >> 4);
            ldsm_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], sQ + swz<D>(r, ch));
          }
        }
        const uint16_t* bk = sK + buf * kBN * D;
        const uint16_t* bv = sV + buf * kBN * D;
        float s[kBN / 8][4];
#pragma unroll
        for (int i = 0; i < kBN / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
          for (int np = 0; np < kBN / 16; ++np) {
            uint32_t b0, b1, b2, b3;
            const int n = np * 16 + (lane & 7) + 8 * (lane >> 4);
            const int ch = 2 * kk + ((lane >> 3) & 1);
            ldsm_x4(b0, b1, b2, b3, bk + swz<D>(n, ch));
            mma_bf16_16816(s[2 * np], qa[kk], b0, b1);
            mma_bf16_16816(s[2 * np + 1], qa[kk], b2, b3);
          }
        }
        // mask + scale (base 2), row maxima
        const int kbase = klo + j * kBN + 2 * (lane & 3);
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int nb = 0; nb < kBN / 8; ++nb) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = kbase + nb * 8 + e;
            float xa = s[nb][e] * scale_log2;
            float xb = s[nb][2 + e] * scale_log2;
            xa = (key >= lo_a && key < hi_a) ? xa : -INFINITY;
            xb = (key >= lo_b && key < hi_b) ? xb : -INFINITY;
            s[nb][e] = xa;
            s[nb][2 + e] = xb;
            mx_a = fmaxf(mx_a, xa);
            mx_b = fmaxf(mx_b, xb);
          }
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float use_a = (mn_a == -INFINITY) ? 0.f : mn_a;
        const float use_b = (mn_b == -INFINITY) ? 0.f : mn_b;
        const float al_a = fast_exp2(m_a - use_a), al_b = fast_exp2(m_b - use_b);
        m_a = mn_a;
        m_b = mn_b;
        float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
        for (int nb = 0; nb < kBN / 8; ++nb) {
          s[nb][0] = fast_exp2(s[nb][0] - use_a);
          s[nb][1] = fast_exp2(s[nb][1] - use_a);
          s[nb][2] = fast_exp2(s[nb][2] - use_b);
          s[nb][3] = fast_exp2(s[nb][3] - use_b);
          sum_a += s[nb][0] + s[nb][1];
          sum_b += s[nb][2] + s[nb][3];
        }
        l_a = l_a * al_a + sum_a;
        l_b = l_b * al_b + sum_b;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          o[i][0] *= al_a;
          o[i][1] *= al_a;
          o[i][2] *= al_b;
          o[i][3] *= al_b;
        }
        // O += P V
#pragma unroll
        for (int kk2 = 0; kk2 < kBN / 16; ++kk2) {
          uint32_t pa[4];
          pa[0] = pack_bf16(s[2 * kk2][0], s[2 * kk2][1]);
          pa[1] = pack_bf16(s[2 * kk2][2], s[2 * kk2][3]);
          pa[2] = pack_bf16(s[2 * kk2 + 1][0], s[2 * kk2 + 1][1]);
          pa[3] = pack_bf16(s[2 * kk2 + 1][2], s[2 * kk2 + 1][3]);
#pragma unroll
          for (int dp = 0; dp < D / 16; ++dp) {
            uint32_t b0, b1, b2, b3;
            const int key = kk2 * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ch = 2 * dp + (lane >> 4);
            ldsm_x4_t(b0, b1, b2, b3, bv + swz<D>(key, ch));
            mma_bf16_16816(o[2 * dp], pa, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
          }
        }
        __syncthreads();  // buffer `buf` is refilled two iterations later
      }
      cp_async_wait<0>();

      // finish the row sums across the quad and write the partial records
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      const int row_a = sRow[ra], row_b = sRow[rb];
      const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
      const float inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
      const int col0 = 2 * (lane & 3);
      if (row_a >= 0) {
        float* dst = part_o + size_t(row_a) * D + col0;
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb)
          *reinterpret_cast<float2*>(dst + nb * 8) = make_float2(o[nb][0] * inv_a, o[nb][1] * inv_a);
        if ((lane & 3) == 0) {
          part_m[row_a] = (l_a > 0.f) ? m_a * kLn2 : -INFINITY;
          part_l[row_a] = l_a;
        }
      }
      if (row_b >= 0) {
        float* dst = part_o + size_t(row_b) * D + col0;
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb)
          *reinterpret_cast<float2*>(dst + nb * 8) = make_float2(o[nb][2] * inv_b, o[nb][3] * inv_b);
        if ((lane & 3) == 0) {
          part_m[row_b] = (l_b > 0.f) ? m_b * kLn2 : -INFINITY;
          part_l[row_b] = l_b;
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) p.timers[w * 2 + 1] = global_timer_ns();
}

template <int D>
cudaError_t launch_fwd_d(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         float scale, float* po, float* pm, float* pl, cudaStream_t s) {
  const size_t smem = fwd_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(fwd_partial_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  fwd_partial_mma_kernel<D><<<p.W, kThreads, smem, s>>>(p, q, k, v, scale * kLog2e, po, pm, pl);
  return cudaGetLastError();
}

}  // namespace

bool fwd_sm100_supported(const DevPlan& p);
cudaError_t launch_fwd_partial_sm100(const DevPlan& p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     float scale, void* part_o, float* part_m, float* part_l, cudaStream_t s);
bool bwd_sm100_supported(const DevPlan& p);

namespace {
bool env_is_mma(const char* name) {
  const char* e = std::getenv(name);
  return e != nullptr && std::strcmp(e, "mma") == 0;
}
}  // namespace

bool tcgen05_supported(const DevPlan& p) {
  static const bool forced = env_is_mma("SPLITKV_FWD_KERNEL") || env_is_mma("SPLITKV_BWD_KERNEL");
  return !forced && fwd_sm100_supported(p) && bwd_sm100_supported(p);
}

// The tcgen05 kernel serves head_dim 128 with G * bs a multiple of 8; every
// other shape runs the mma.sync kernel.  SPLITKV_FWD_KERNEL=mma selects the
// mma.sync kernel for every shape (for comparisons).
cudaError_t launch_fwd_partial(const DevPlan& p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, float scale, void* part_o, float* part_m,
                               float* part_l, cudaStream_t s) {
  static const bool force_mma = env_is_mma("SPLITKV_FWD_KERNEL");
  if (!force_mma && fwd_sm100_supported(p))
    return launch_fwd_partial_sm100(p, q, k, v, scale, part_o, part_m, part_l, s);
  if (p.partial_bf16 || p.dynamic) return cudaErrorNotSupported;   // the entry points check this first
  float* po = static_cast<float*>(part_o);
  if (p.d == 64) return launch_fwd_d<64>(p, q, k, v, scale, po, part_m, part_l, s);
  return launch_fwd_d<128>(p, q, k, v, scale, po, part_m, part_l, s);
}

}  // namespace splitkv
