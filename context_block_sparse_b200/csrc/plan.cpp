// Host planner: anchor-block mask metadata and cost-aware LPT schedules.
//
// Source: "Split-KV: Efficient Context Parallelism for Training Diffusion
// Drafters" (digest page, Abstract) and the news page "Split-KV speeds
// diffusion drafter training by keeping long-context data local", sections
// "Why short queries change the problem" (the mask: own-sample preceding
// context plus the block's own tokens) and "Balance actual attention work"
// (chunk cost = realised attention usage; LPT = sort by cost, give each chunk
// to the least-loaded eligible worker, optionally keeping counts equal).
//
// Everything here is integer arithmetic, so schedules are reproducible bit
// for bit.  The worker choice uses a binary heap keyed by (load, worker id).
#include <algorithm>
#include <chrono>
#include <cstring>
#include <new>
#include <vector>

#include "splitkv.h"
#include "splitkv_internal.h"

using splitkv::DevPlan;

namespace {

struct I4 {
  int32_t x, y, z, w;
};

struct Item {
  int32_t c, g, slice, t0, t1;
  uint64_t cost;
};

}  // namespace

// Largest wait limit a plan accepts (a minute): a wait that long has failed.
constexpr int64_t kMaxWaitLimitNs = 60000000000LL;

struct splitkv_plan_s {
  // problem
  int32_t S = 0, A = 0, bs = 0, Hq = 0, Hkv = 0, d = 0, C = 0, W = 0, Wb = 0, q_slice = 0;
  uint32_t flags = 0;
  std::vector<int32_t> lens, anchors;
  // derived
  int64_t N = 0, Nq = 0;
  int32_t G = 0, num_chunks = 0, blocks_per_tile = 0;
  std::vector<int32_t> block_lo, block_hi;        // per block: [S_s, a_b)
  std::vector<I4> entries;                         // {block, lo, hi, chunk}
  std::vector<int32_t> chunk_entry_ptr;            // [num_chunks + 1]
  std::vector<I4> tiles;                           // {e0, e1, klo, khi}
  std::vector<int32_t> chunk_tile_ptr;             // [num_chunks + 1]
  std::vector<uint64_t> chunk_pairs;               // per query head
  std::vector<Item> fwd_items, bwd_items;          // non-zero-cost items
  std::vector<int32_t> fwd_worker_ptr, bwd_worker_ptr;
  std::vector<int32_t> fwd_order, bwd_order;       // item indices grouped by worker
  std::vector<int32_t> fwd_lpt, bwd_lpt;           // item indices in LPT order (cost desc, index asc)
  std::vector<uint64_t> fwd_loads, bwd_loads, contig_loads;
  std::vector<int32_t> block_entry_ptr, block_entries;
  std::vector<int32_t> zero_chunks;
  // ranks (splitkv_plan_shard): this plan holds the entries of the chunks rank `rank`
  // owns and the in-block term of blocks [bt_lo, bt_hi); a plain plan is rank 0 of 1
  int32_t R = 1, rank = 0, bt_lo = 0, bt_hi = 0;
  std::vector<int32_t> chunk_owner;               // [num_chunks]
  double plan_us = 0.0;
  // device copy
  void* d_blob = nullptr;
  size_t d_cap = 0;
  void* h_pinned = nullptr;
  size_t h_cap = 0;
  cudaEvent_t upload_ev = nullptr;
  bool upload_pending = false;
  bool uploaded = false;
  int64_t wait_limit_ns = 2000000000LL;            // splitkv_plan_set_wait_limit
  DevPlan dev{};
};

namespace {

int validate(const splitkv_problem* p) {
  if (!p || !p->sample_lens || !p->anchors) return SPLITKV_ERR_INVALID_ARG;
  if (p->num_samples < 1 || p->num_anchors < 1 || p->block_size < 1 || p->num_q_heads < 1 ||
      p->num_kv_heads < 1 || p->head_dim < 1 || p->kv_chunk < 1 || p->num_workers < 1 ||
      p->num_bwd_workers < 0 || p->q_slice < 0)
    return SPLITKV_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads) return SPLITKV_ERR_INVALID_ARG;
  if (p->flags & ~uint32_t(SPLITKV_FLAG_EQUAL_COUNT | SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT | SPLITKV_FLAG_PARTIAL_BF16 |
                           SPLITKV_FLAG_TILE_COST | SPLITKV_FLAG_FWD_TILE_COST | SPLITKV_FLAG_DYNAMIC_CLAIM |
                           SPLITKV_FLAG_CONTIGUOUS_SCHEDULE | SPLITKV_FLAG_CONTIGUOUS_RANKS))
    return SPLITKV_ERR_INVALID_ARG;
  if ((p->flags & SPLITKV_FLAG_CONTIGUOUS_SCHEDULE) &&
      (p->flags & (SPLITKV_FLAG_EQUAL_COUNT | SPLITKV_FLAG_DYNAMIC_CLAIM)))
    return SPLITKV_ERR_INVALID_ARG;
  int64_t N = 0;
  for (int s = 0; s < p->num_samples; ++s) {
    if (p->sample_lens[s] < 1) return SPLITKV_ERR_INVALID_ARG;
    N += p->sample_lens[s];
  }
  if (N >= (int64_t(1) << 31)) return SPLITKV_ERR_INVALID_ARG;
  for (int b = 0; b < p->num_anchors; ++b)
    if (p->anchors[b] < 0 || p->anchors[b] >= N) return SPLITKV_ERR_INVALID_ARG;
  const int64_t G = p->num_q_heads / p->num_kv_heads;
  if (G * p->block_size > splitkv::kTileRows || splitkv::kTileRows % (G * p->block_size))
    return SPLITKV_ERR_UNSUPPORTED;
  if (int64_t(p->num_anchors) * p->block_size >= (int64_t(1) << 31)) return SPLITKV_ERR_INVALID_ARG;
  return SPLITKV_OK;
}

// LPT: items sorted by (cost desc, chunk, head, slice asc); each to the eligible
// worker of minimum (load, id).  Items are generated in (chunk, head, slice)
// order, so a stable sort on cost alone gives that order.  The workers sit in a
// binary min-heap keyed by (load, id); eligibility is monotone (a worker that
// stops being eligible never becomes eligible again), so an ineligible top is
// removed for good.
// Item indices by cost descending, equal costs in index order: an LSD radix sort on
// the complemented cost, one stable counting pass per byte that differs between
// keys (the same order as a stable sort by cost descending, in O(n) per pass).
void sort_by_cost_desc(const std::vector<Item>& items, std::vector<int32_t>& out) {
  const int64_t n = int64_t(items.size());
  uint64_t max_cost = 0;
  for (const Item& it : items) max_cost = std::max(max_cost, it.cost);
  if (max_cost <= 0xffffffffull && n <= (int64_t(1) << 31)) {
    // costs fit in 32 bits: sort packed keys ((~cost) << 32 | index) by their high half,
    // stably, so equal costs keep index order -- one contiguous array, no indirection
    std::vector<uint64_t> a(static_cast<size_t>(n)), b(static_cast<size_t>(n));
    uint32_t any_one = 0, all_one = 0xffffffffu;
    for (int64_t i = 0; i < n; ++i) {
      const uint32_t k = ~uint32_t(items[size_t(i)].cost);
      any_one |= k;
      all_one &= k;
      a[size_t(i)] = (uint64_t(k) << 32) | uint64_t(i);
    }
    for (int shift = 32; shift < 64; shift += 8) {
      if ((((uint64_t(any_one ^ all_one) << 32) >> shift) & 0xffu) == 0) continue;   // a constant byte
      int64_t cnt[257] = {};
      for (int64_t i = 0; i < n; ++i) cnt[((a[size_t(i)] >> shift) & 0xffu) + 1]++;
      for (int d = 0; d < 256; ++d) cnt[d + 1] += cnt[d];
      for (int64_t i = 0; i < n; ++i) b[size_t(cnt[(a[size_t(i)] >> shift) & 0xffu]++)] = a[size_t(i)];
      a.swap(b);
    }
    out.resize(size_t(n));
    for (int64_t i = 0; i < n; ++i) out[size_t(i)] = int32_t(a[size_t(i)] & 0xffffffffu);
    return;
  }
  std::vector<int32_t> a(n), b(n);
  for (int64_t i = 0; i < n; ++i) a[i] = int32_t(i);
  uint64_t any_one = 0, all_one = ~uint64_t(0);
  for (const Item& it : items) {
    any_one |= ~it.cost;
    all_one &= ~it.cost;
  }
  for (int shift = 0; shift < 64; shift += 8) {
    if ((((any_one ^ all_one) >> shift) & 0xffu) == 0) continue;   // the same byte in every key
    int64_t cnt[257] = {};
    for (int64_t i = 0; i < n; ++i) cnt[((~items[a[i]].cost >> shift) & 0xffu) + 1]++;
    for (int d = 0; d < 256; ++d) cnt[d + 1] += cnt[d];
    for (int64_t i = 0; i < n; ++i) b[cnt[(~items[a[i]].cost >> shift) & 0xffu]++] = a[i];
    a.swap(b);
  }
  out.swap(a);
}

// The contiguous ("unbalanced") schedule: items in their (chunk, head, slice) order,
// item i of n to worker floor(i W / n); `order` lists them worker by worker (which is
// item order), and `sorted` receives the same order.
void contiguous_schedule(const std::vector<Item>& items, int W, std::vector<int32_t>& worker_ptr,
                         std::vector<int32_t>& order, std::vector<uint64_t>& loads, std::vector<int32_t>& sorted) {
  const int64_t n = int64_t(items.size());
  loads.assign(size_t(W), 0);
  worker_ptr.assign(size_t(W) + 1, 0);
  order.resize(size_t(n));
  for (int64_t i = 0; i < n; ++i) {
    const int64_t w = (i * W) / n;
    loads[size_t(w)] += items[size_t(i)].cost;
    worker_ptr[size_t(w) + 1]++;
    order[size_t(i)] = int32_t(i);
  }
  for (int w = 0; w < W; ++w) worker_ptr[size_t(w) + 1] += worker_ptr[size_t(w)];
  sorted = order;
}

void lpt_schedule(const std::vector<Item>& items, int W, bool equal_count,
                  std::vector<int32_t>& worker_ptr, std::vector<int32_t>& order,
                  std::vector<uint64_t>& loads, std::vector<int32_t>& sorted) {
  const int64_t n = int64_t(items.size());
  sort_by_cost_desc(items, sorted);
  const int64_t q = n / W, r = n % W;
  loads.assign(W, 0);
  std::vector<int64_t> counts(W, 0);
  std::vector<int32_t> owner(n);
  // heap of worker ids ordered by (load, id)
  std::vector<int32_t> heap(W);
  for (int w = 0; w < W; ++w) heap[w] = w;   // all loads 0: ids ascending is a valid heap
  int hn = W;
  auto less = [&](int32_t a, int32_t b) { return loads[a] != loads[b] ? loads[a] < loads[b] : a < b; };
  auto sift_down = [&](int i) {
    const int32_t x = heap[i];
    for (;;) {
      int c = 2 * i + 1;
      if (c >= hn) break;
      if (c + 1 < hn && less(heap[c + 1], heap[c])) ++c;
      if (!less(heap[c], x)) break;
      heap[i] = heap[c];
      i = c;
    }
    heap[i] = x;
  };
  int64_t n_full = 0;  // workers holding q + 1 items
  // Plain LPT whose loads stay small enough: the heap holds keys (load << id_bits) | id,
  // whose integer order is the (load, id) order, and the sift picks children without
  // branches.  Distinct keys have one minimum, so every choice is the same as below.
  int id_bits = 1;
  while ((int64_t(1) << id_bits) < W) ++id_bits;
  uint64_t total = 0;
  bool fits = !equal_count;
  for (const Item& it : items) {
    total += it.cost;
    if (total >= (uint64_t(1) << (63 - id_bits))) fits = false;
  }
  if (fits) {
    std::vector<uint64_t> key(static_cast<size_t>(W));
    for (int w = 0; w < W; ++w) key[size_t(w)] = uint64_t(w);   // all loads 0: ids ascending is a heap
    const uint64_t id_mask = (uint64_t(1) << id_bits) - 1;
    for (int64_t k = 0; k < n; ++k) {
      const int32_t it = sorted[size_t(k)];
      const uint64_t top = key[0];
      const int32_t w = int32_t(top & id_mask);
      const uint64_t x = top + (items[size_t(it)].cost << id_bits);
      loads[size_t(w)] += items[size_t(it)].cost;
      owner[size_t(k)] = w;
      int i = 0;
      for (;;) {
        int c = 2 * i + 1;
        if (c >= W) break;
        uint64_t kc = key[size_t(c)];
        if (c + 1 < W) {
          const uint64_t k2 = key[size_t(c) + 1];
          const bool right = k2 < kc;
          c += right ? 1 : 0;
          kc = right ? k2 : kc;
        }
        if (kc >= x) break;
        key[size_t(i)] = kc;
        i = c;
      }
      key[size_t(i)] = x;
    }
  }
  for (int64_t k = 0; k < n && !fits; ++k) {
    const int32_t it = sorted[k];
    if (equal_count) {
      // drop tops that can no longer take an item; some worker always can
      for (;;) {
        const int32_t c = heap[0];
        if (counts[c] < q || (counts[c] == q && n_full < r)) break;
        heap[0] = heap[--hn];
        sift_down(0);
      }
    }
    const int32_t w = heap[0];
    loads[w] += items[it].cost;
    counts[w] += 1;
    if (counts[w] == q + 1) ++n_full;
    owner[k] = w;
    sift_down(0);   // only the top's key grew
  }
  // group by worker, keeping assignment order
  worker_ptr.assign(W + 1, 0);
  for (int64_t k = 0; k < n; ++k) worker_ptr[owner[k] + 1]++;
  for (int w = 0; w < W; ++w) worker_ptr[w + 1] += worker_ptr[w];
  order.resize(n);
  std::vector<int32_t> fill(worker_ptr.begin(), worker_ptr.end() - 1);
  for (int64_t k = 0; k < n; ++k) order[fill[owner[k]]++] = sorted[k];
}

int build(splitkv_plan_t* P, const splitkv_problem* p) {
  const auto clock_start = std::chrono::steady_clock::now();
  int st = validate(p);
  if (st != SPLITKV_OK) return st;
  P->S = p->num_samples;
  P->A = p->num_anchors;
  P->bs = p->block_size;
  P->Hq = p->num_q_heads;
  P->Hkv = p->num_kv_heads;
  P->d = p->head_dim;
  P->C = p->kv_chunk;
  P->W = p->num_workers;
  P->Wb = p->num_bwd_workers > 0 ? p->num_bwd_workers : p->num_workers;
  P->q_slice = p->q_slice;
  P->flags = p->flags;
  P->lens.assign(p->sample_lens, p->sample_lens + P->S);
  P->anchors.assign(p->anchors, p->anchors + P->A);
  P->G = P->Hq / P->Hkv;
  P->blocks_per_tile = splitkv::kTileRows / (P->G * P->bs);

  // sample starts; block intervals [S_s, a_b) by binary search over the starts
  // (reading B of the block keys: [S_s, min(a_b + bs, S_s + L_s)))
  std::vector<int64_t> starts(P->S + 1, 0);
  for (int s = 0; s < P->S; ++s) starts[s + 1] = starts[s] + P->lens[s];
  P->N = starts[P->S];
  P->Nq = int64_t(P->A) * P->bs;
  P->num_chunks = int32_t((P->N + P->C - 1) / P->C);
  P->block_lo.resize(P->A);
  P->block_hi.resize(P->A);
  for (int b = 0; b < P->A; ++b) {
    const int64_t a = P->anchors[b];
    const int s = int(std::upper_bound(starts.begin(), starts.end(), a) - starts.begin()) - 1;
    P->block_lo[b] = int32_t(starts[s]);
    P->block_hi[b] = (P->flags & SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT)
                         ? int32_t(std::min<int64_t>(a + P->bs, starts[s + 1]))
                         : int32_t(a);
  }

  // entries: each block's interval covers chunks lo/C .. (hi-1)/C; bucket by chunk
  std::vector<int32_t> cnt(P->num_chunks + 1, 0);
  for (int b = 0; b < P->A; ++b) {
    const int lo = P->block_lo[b], hi = P->block_hi[b];
    if (lo >= hi) continue;
    for (int c = lo / P->C; c <= (hi - 1) / P->C; ++c) cnt[c + 1]++;
  }
  P->chunk_entry_ptr.assign(P->num_chunks + 1, 0);
  for (int c = 0; c < P->num_chunks; ++c) P->chunk_entry_ptr[c + 1] = P->chunk_entry_ptr[c] + cnt[c + 1];
  const int32_t E = P->chunk_entry_ptr[P->num_chunks];
  P->entries.resize(size_t(E));
  {
    std::vector<int32_t> fill(P->chunk_entry_ptr.begin(), P->chunk_entry_ptr.end() - 1);
    for (int b = 0; b < P->A; ++b) {
      const int lo = P->block_lo[b], hi = P->block_hi[b];
      if (lo >= hi) continue;
      for (int c = lo / P->C; c <= (hi - 1) / P->C; ++c) {
        const int c0 = c * P->C;
        const int c1 = int(std::min<int64_t>(int64_t(c0) + P->C, P->N));
        P->entries[fill[c]++] = I4{b, std::max(lo, c0), std::min(hi, c1), c};
      }
    }
  }
  P->chunk_pairs.assign(P->num_chunks, 0);
  for (int c = 0; c < P->num_chunks; ++c) {
    auto first = P->entries.begin() + P->chunk_entry_ptr[c];
    auto last = P->entries.begin() + P->chunk_entry_ptr[c + 1];
    std::sort(first, last, [](const I4& a, const I4& b) {
      if (a.y != b.y) return a.y < b.y;
      if (a.z != b.z) return a.z < b.z;
      return a.x < b.x;
    });
    uint64_t keys = 0;
    for (auto it = first; it != last; ++it) keys += uint64_t(it->z - it->y);
    P->chunk_pairs[c] = keys * uint64_t(P->bs);
  }

  // ranks: whole chunks to ranks by LPT with equal counts (the pages' device rule), every
  // chunk an item -- zero-cost ones too, since its keys live somewhere -- of cost
  // Hq * pairs_c (or, under SPLITKV_FLAG_CONTIGUOUS_RANKS, chunk c to rank floor(c R / n));
  // then keep this rank's entries (their pairs are the rank's work) and the in-block
  // term of its contiguous block range [floor(r A / R), floor((r + 1) A / R))
  P->chunk_owner.assign(size_t(P->num_chunks), 0);
  P->bt_lo = int32_t(int64_t(P->rank) * P->A / P->R);
  P->bt_hi = int32_t(int64_t(P->rank + 1) * P->A / P->R);
  if (P->R > 1 && (P->flags & SPLITKV_FLAG_CONTIGUOUS_RANKS)) {
    for (int c = 0; c < P->num_chunks; ++c)
      P->chunk_owner[size_t(c)] = int32_t((int64_t(c) * P->R) / P->num_chunks);
  } else if (P->R > 1) {
    std::vector<Item> chunk_items(size_t(P->num_chunks));
    for (int c = 0; c < P->num_chunks; ++c)
      chunk_items[size_t(c)] = Item{c, 0, 0, 0, 0, P->chunk_pairs[size_t(c)] * uint64_t(P->Hq)};
    std::vector<int32_t> rank_ptr, rank_order, by_cost;
    std::vector<uint64_t> rank_loads;
    lpt_schedule(chunk_items, P->R, true, rank_ptr, rank_order, rank_loads, by_cost);
    for (int r = 0; r < P->R; ++r)
      for (int k = rank_ptr[size_t(r)]; k < rank_ptr[size_t(r) + 1]; ++k)
        P->chunk_owner[size_t(chunk_items[size_t(rank_order[size_t(k)])].c)] = r;
  }
  if (P->R > 1) {
    std::vector<I4> kept;
    std::vector<int32_t> kept_ptr(size_t(P->num_chunks) + 1, 0);
    for (int c = 0; c < P->num_chunks; ++c) {
      if (P->chunk_owner[size_t(c)] == P->rank)
        kept.insert(kept.end(), P->entries.begin() + P->chunk_entry_ptr[size_t(c)],
                    P->entries.begin() + P->chunk_entry_ptr[size_t(c) + 1]);
      else
        P->chunk_pairs[size_t(c)] = 0;
      kept_ptr[size_t(c) + 1] = int32_t(kept.size());
    }
    P->entries.swap(kept);
    P->chunk_entry_ptr.swap(kept_ptr);
  }
  const int32_t E_kept = int32_t(P->entries.size());

  // 128-row query tiles of consecutive entries inside each chunk
  P->tiles.clear();
  P->chunk_tile_ptr.assign(P->num_chunks + 1, 0);
  for (int c = 0; c < P->num_chunks; ++c) {
    P->chunk_tile_ptr[c] = int32_t(P->tiles.size());
    for (int e0 = P->chunk_entry_ptr[c]; e0 < P->chunk_entry_ptr[c + 1]; e0 += P->blocks_per_tile) {
      const int e1 = std::min(e0 + P->blocks_per_tile, P->chunk_entry_ptr[c + 1]);
      int klo = P->entries[e0].y, khi = P->entries[e0].z;
      for (int e = e0; e < e1; ++e) {
        klo = std::min(klo, P->entries[e].y);
        khi = std::max(khi, P->entries[e].z);
      }
      P->tiles.push_back(I4{e0, e1, klo, khi});
    }
  }
  P->chunk_tile_ptr[P->num_chunks] = int32_t(P->tiles.size());

  // work items: per (chunk, KV head), optionally cut into slices of q_slice tiles
  auto tile_cost = [&](int t) {
    uint64_t keys = 0;
    for (int e = P->tiles[t].x; e < P->tiles[t].y; ++e) keys += uint64_t(P->entries[e].z - P->entries[e].y);
    return keys * uint64_t(P->bs) * uint64_t(P->G);
  };
  // tile cost of the backward schedule (SPLITKV_FLAG_TILE_COST): executed (row, key)
  // pairs of whole tile steps of the dK/dV kernel, whose key tiles hold 128 keys
  constexpr int kKeyTile = 128;
  const bool by_tiles = (P->flags & SPLITKV_FLAG_TILE_COST) != 0;
  const uint64_t step_pairs = uint64_t(splitkv::kTileRows) * uint64_t(kKeyTile);
  auto bwd_exec = [&](int c, int t0, int t1) {   // per key tile of chunk c, the tiles that meet it
    const int64_t c0 = int64_t(c) * P->C, c1 = std::min<int64_t>(c0 + P->C, P->N);
    uint64_t steps = 0;
    for (int64_t k0 = c0; k0 < c1; k0 += kKeyTile)
      for (int t = t0; t < t1; ++t)
        if (P->tiles[t].z < k0 + kKeyTile && P->tiles[t].w > k0) ++steps;
    return steps * step_pairs;
  };
  // tile cost of the forward schedule (SPLITKV_FLAG_FWD_TILE_COST): the forward
  // kernel runs tiles t0, t0 + 1 (then t0 + 2, t0 + 3, ...) together over the key
  // tiles of their joint key range
  const bool fwd_by_tiles = (P->flags & SPLITKV_FLAG_FWD_TILE_COST) != 0;
  auto fwd_exec = [&](int t0, int t1) {
    uint64_t steps = 0;
    for (int t = t0; t < t1; t += 2) {
      const int n = std::min(2, t1 - t);
      int klo = P->tiles[t].z, khi = P->tiles[t].w;
      if (n == 2) {
        klo = std::min(klo, P->tiles[t + 1].z);
        khi = std::max(khi, P->tiles[t + 1].w);
      }
      steps += uint64_t(n) * uint64_t((int64_t(khi) - klo + kKeyTile - 1) / kKeyTile);
    }
    return steps * step_pairs;
  };
  P->fwd_items.clear();
  P->bwd_items.clear();
  P->zero_chunks.clear();
  // at most one forward item per tile and KV head, one backward item per chunk and KV head
  P->fwd_items.reserve(P->tiles.size() * size_t(P->Hkv));
  P->bwd_items.reserve(size_t(P->num_chunks) * size_t(P->Hkv));
  for (int c = 0; c < P->num_chunks; ++c) {
    const int t0 = P->chunk_tile_ptr[c], t1 = P->chunk_tile_ptr[c + 1];
    if (t0 == t1) {
      if (P->chunk_owner[size_t(c)] == P->rank) P->zero_chunks.push_back(c);   // other ranks' keys: not ours
      continue;
    }
    const uint64_t whole = P->chunk_pairs[c] * uint64_t(P->G);
    const uint64_t bcost = by_tiles ? bwd_exec(c, t0, t1) : whole;
    for (int g = 0; g < P->Hkv; ++g) P->bwd_items.push_back(Item{c, g, 0, t0, t1, bcost});
    if (P->q_slice <= 0) {
      const uint64_t fcost = fwd_by_tiles ? fwd_exec(t0, t1) : whole;
      for (int g = 0; g < P->Hkv; ++g) P->fwd_items.push_back(Item{c, g, 0, t0, t1, fcost});
    } else {
      // generated in (chunk, head, slice) order: the LPT sort relies on it for ties
      const size_t first = P->fwd_items.size();
      int slice = 0;
      for (int s0 = t0; s0 < t1; s0 += P->q_slice, ++slice) {
        const int s1 = std::min(s0 + P->q_slice, t1);
        uint64_t cost = 0;
        if (fwd_by_tiles)
          cost = fwd_exec(s0, s1);
        else
          for (int t = s0; t < s1; ++t) cost += tile_cost(t);
        P->fwd_items.push_back(Item{c, 0, slice, s0, s1, cost});
      }
      const size_t ns = P->fwd_items.size() - first;
      for (int g = 1; g < P->Hkv; ++g)
        for (size_t i = 0; i < ns; ++i) {
          Item it = P->fwd_items[first + i];
          it.g = g;
          P->fwd_items.push_back(it);
        }
    }
  }
  // drop zero-cost items (cannot occur: every tile holds a non-empty interval)
  auto nonzero = [](std::vector<Item>& v) {
    v.erase(std::remove_if(v.begin(), v.end(), [](const Item& it) { return it.cost == 0; }), v.end());
  };
  nonzero(P->fwd_items);
  nonzero(P->bwd_items);
  const bool eq = (P->flags & SPLITKV_FLAG_EQUAL_COUNT) != 0;
  if (P->flags & SPLITKV_FLAG_CONTIGUOUS_SCHEDULE) {
    contiguous_schedule(P->fwd_items, P->W, P->fwd_worker_ptr, P->fwd_order, P->fwd_loads, P->fwd_lpt);
    contiguous_schedule(P->bwd_items, P->Wb, P->bwd_worker_ptr, P->bwd_order, P->bwd_loads, P->bwd_lpt);
  } else {
    lpt_schedule(P->fwd_items, P->W, eq, P->fwd_worker_ptr, P->fwd_order, P->fwd_loads, P->fwd_lpt);
    lpt_schedule(P->bwd_items, P->Wb, eq, P->bwd_worker_ptr, P->bwd_order, P->bwd_loads, P->bwd_lpt);
  }

  // contiguous ("unbalanced") baseline: the num_chunks * Hkv (chunk, head) items in
  // order, item i to worker floor(i W / n), zero-cost items included
  P->contig_loads.assign(P->W, 0);
  {
    const int64_t n = int64_t(P->num_chunks) * P->Hkv;
    for (int64_t i = 0; i < n; ++i) {
      const int64_t c = i / P->Hkv;
      P->contig_loads[size_t((i * P->W) / n)] += P->chunk_pairs[c] * uint64_t(P->G);
    }
  }

  // block -> entries (ascending chunk)
  P->block_entry_ptr.assign(P->A + 1, 0);
  for (int e = 0; e < E_kept; ++e) P->block_entry_ptr[P->entries[e].x + 1]++;
  for (int b = 0; b < P->A; ++b) P->block_entry_ptr[b + 1] += P->block_entry_ptr[b];
  P->block_entries.assign(size_t(E_kept), 0);
  {
    std::vector<int32_t> fill(P->block_entry_ptr.begin(), P->block_entry_ptr.end() - 1);
    for (int e = 0; e < E_kept; ++e) P->block_entries[fill[P->entries[e].x]++] = e;  // e ascends with chunk
  }
  P->uploaded = false;
  P->plan_us = std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now() - clock_start).count();
  return SPLITKV_OK;
}

double imbalance(const std::vector<uint64_t>& loads) {
  if (loads.empty()) return 0.0;
  long double total = 0;
  uint64_t mx = 0;
  for (uint64_t x : loads) {
    total += x;
    mx = std::max(mx, x);
  }
  if (total == 0) return 0.0;
  return double(mx / (total / loads.size()) - 1.0L);
}

}  // namespace

extern "C" {

const char* splitkv_error_string(int status) {
  switch (status) {
    case SPLITKV_OK: return "ok";
    case SPLITKV_ERR_INVALID_ARG: return "invalid argument";
    case SPLITKV_ERR_UNSUPPORTED: return "unsupported shape";
    case SPLITKV_ERR_WORKSPACE_TOO_SMALL: return "buffer or workspace too small";
    case SPLITKV_ERR_CUDA: return "CUDA runtime error";
    case SPLITKV_ERR_TIMEOUT: return "device wait timed out";
    case SPLITKV_ERR_NOT_UPLOADED: return "plan has no device copy (call splitkv_plan_upload)";
    case SPLITKV_ERR_NO_MEMORY: return "out of memory";
    default: return "unknown status";
  }
}

int splitkv_plan(const splitkv_problem* problem, splitkv_plan_t** out) {
  if (!out) return SPLITKV_ERR_INVALID_ARG;
  *out = nullptr;
  splitkv_plan_t* P = nullptr;
  try {
    P = new splitkv_plan_t();
    const int st = build(P, problem);
    if (st != SPLITKV_OK) {
      delete P;
      return st;
    }
  } catch (const std::bad_alloc&) {
    delete P;
    return SPLITKV_ERR_NO_MEMORY;
  } catch (...) {
    delete P;
    return SPLITKV_ERR_INVALID_ARG;
  }
  *out = P;
  return SPLITKV_OK;
}

int splitkv_plan_shard(const splitkv_problem* problem, int32_t num_ranks, int32_t rank, splitkv_plan_t** out) {
  if (!out) return SPLITKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_ranks < 1 || rank < 0 || rank >= num_ranks) return SPLITKV_ERR_INVALID_ARG;
  splitkv_plan_t* P = nullptr;
  try {
    P = new splitkv_plan_t();
    P->R = num_ranks;
    P->rank = rank;
    const int st = build(P, problem);
    if (st != SPLITKV_OK) {
      delete P;
      return st;
    }
  } catch (const std::bad_alloc&) {
    delete P;
    return SPLITKV_ERR_NO_MEMORY;
  } catch (...) {
    delete P;
    return SPLITKV_ERR_INVALID_ARG;
  }
  *out = P;
  return SPLITKV_OK;
}

int splitkv_plan_update(splitkv_plan_t* plan, const splitkv_problem* problem) {
  if (!plan) return SPLITKV_ERR_INVALID_ARG;
  const int st0 = validate(problem);
  if (st0 != SPLITKV_OK) return st0;
  if (plan->upload_pending) {
    // the pinned staging buffer may still be read by the previous copy
    if (cudaEventSynchronize(plan->upload_ev) != cudaSuccess) return SPLITKV_ERR_CUDA;
    plan->upload_pending = false;
  }
  try {
    return build(plan, problem);
  } catch (const std::bad_alloc&) {
    return SPLITKV_ERR_NO_MEMORY;
  } catch (...) {
    return SPLITKV_ERR_INVALID_ARG;
  }
}

int splitkv_plan_upload(splitkv_plan_t* P, void* stream) {
  if (!P) return SPLITKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // layout of the blob: tables packed at 256-byte offsets, then the timers
  struct Seg {
    const void* src;
    size_t bytes;
    size_t off;
  };
  std::vector<int32_t> fwd_items, bwd_items;
  auto pack_items = [](const std::vector<Item>& items, const std::vector<int32_t>& order,
                       std::vector<int32_t>& dst) {
    dst.resize(order.size() * 4);
    for (size_t i = 0; i < order.size(); ++i) {
      const Item& it = items[order[i]];
      dst[4 * i + 0] = it.c;
      dst[4 * i + 1] = it.g;
      dst[4 * i + 2] = it.t0;
      dst[4 * i + 3] = it.t1;
    }
  };
  // run-time claims walk the whole lists in LPT order; otherwise each worker's items
  const bool dynamic = (P->flags & SPLITKV_FLAG_DYNAMIC_CLAIM) != 0;
  try {
    pack_items(P->fwd_items, dynamic ? P->fwd_lpt : P->fwd_order, fwd_items);
    pack_items(P->bwd_items, dynamic ? P->bwd_lpt : P->bwd_order, bwd_items);
  } catch (...) {
    return SPLITKV_ERR_NO_MEMORY;
  }
  Seg segs[] = {
      {P->entries.data(), P->entries.size() * sizeof(I4), 0},
      {P->tiles.data(), P->tiles.size() * sizeof(I4), 0},
      {fwd_items.data(), fwd_items.size() * sizeof(int32_t), 0},
      {P->fwd_worker_ptr.data(), P->fwd_worker_ptr.size() * sizeof(int32_t), 0},
      {bwd_items.data(), bwd_items.size() * sizeof(int32_t), 0},
      {P->bwd_worker_ptr.data(), P->bwd_worker_ptr.size() * sizeof(int32_t), 0},
      {P->block_entry_ptr.data(), P->block_entry_ptr.size() * sizeof(int32_t), 0},
      {P->block_entries.data(), P->block_entries.size() * sizeof(int32_t), 0},
      {P->zero_chunks.data(), P->zero_chunks.size() * sizeof(int32_t), 0},
  };
  const int nseg = int(sizeof(segs) / sizeof(segs[0]));
  size_t off = 0;
  for (int i = 0; i < nseg; ++i) {
    segs[i].off = off;
    off = splitkv::align_up(off + segs[i].bytes, 256);
  }
  const size_t table_bytes = off;
  const size_t timer_off = table_bytes;
  const size_t status_off = timer_off + splitkv::align_up(size_t(2 * P->W + P->Wb) * 2 * sizeof(long long), 256);
  const size_t total = status_off + 256;

  if (P->upload_pending) {
    if (cudaEventSynchronize(P->upload_ev) != cudaSuccess) return SPLITKV_ERR_CUDA;
    P->upload_pending = false;
  }
  if (!P->upload_ev) {
    if (cudaEventCreateWithFlags(&P->upload_ev, cudaEventDisableTiming) != cudaSuccess) return SPLITKV_ERR_CUDA;
  }
  if (total > P->d_cap) {
    if (P->d_blob) {
      // kernels queued earlier may still read the old tables
      if (cudaStreamSynchronize(s) != cudaSuccess) return SPLITKV_ERR_CUDA;
      if (cudaDeviceSynchronize() != cudaSuccess) return SPLITKV_ERR_CUDA;
      cudaFree(P->d_blob);
      P->d_blob = nullptr;
      P->d_cap = 0;
    }
    const size_t cap = splitkv::align_up(total + total / 4, 4096);
    if (cudaMalloc(&P->d_blob, cap) != cudaSuccess) {
      cudaGetLastError();
      return SPLITKV_ERR_NO_MEMORY;
    }
    P->d_cap = cap;
    if (cudaMemsetAsync(P->d_blob, 0, cap, s) != cudaSuccess) return SPLITKV_ERR_CUDA;
  }
  if (table_bytes > P->h_cap) {
    if (P->h_pinned) cudaFreeHost(P->h_pinned);
    P->h_pinned = nullptr;
    P->h_cap = 0;
    const size_t cap = splitkv::align_up(table_bytes + table_bytes / 4 + 256, 4096);
    if (cudaHostAlloc(&P->h_pinned, cap, cudaHostAllocDefault) != cudaSuccess) {
      cudaGetLastError();
      return SPLITKV_ERR_NO_MEMORY;
    }
    P->h_cap = cap;
  }
  char* h = static_cast<char*>(P->h_pinned);
  for (int i = 0; i < nseg; ++i)
    if (segs[i].bytes) std::memcpy(h + segs[i].off, segs[i].src, segs[i].bytes);
  if (table_bytes &&
      cudaMemcpyAsync(P->d_blob, P->h_pinned, table_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return SPLITKV_ERR_CUDA;
  if (cudaEventRecord(P->upload_ev, s) != cudaSuccess) return SPLITKV_ERR_CUDA;
  P->upload_pending = true;

  char* d = static_cast<char*>(P->d_blob);
  DevPlan& v = P->dev;
  v.entries = reinterpret_cast<const int4*>(d + segs[0].off);
  v.tiles = reinterpret_cast<const int4*>(d + segs[1].off);
  v.fwd_items = reinterpret_cast<const int4*>(d + segs[2].off);
  v.fwd_worker_ptr = reinterpret_cast<const int*>(d + segs[3].off);
  v.bwd_items = reinterpret_cast<const int4*>(d + segs[4].off);
  v.bwd_worker_ptr = reinterpret_cast<const int*>(d + segs[5].off);
  v.block_entry_ptr = reinterpret_cast<const int*>(d + segs[6].off);
  v.block_entries = reinterpret_cast<const int*>(d + segs[7].off);
  v.zero_chunks = reinterpret_cast<const int*>(d + segs[8].off);
  v.timers = reinterpret_cast<long long*>(d + timer_off);
  v.status = reinterpret_cast<int*>(d + status_off);
  v.num_zero_chunks = int(P->zero_chunks.size());
  v.N = int(P->N);
  v.Nq = int(P->Nq);
  v.A = P->A;
  v.bs = P->bs;
  v.Hq = P->Hq;
  v.Hkv = P->Hkv;
  v.G = P->G;
  v.d = P->d;
  v.C = P->C;
  v.num_chunks = P->num_chunks;
  v.E = int(P->entries.size());
  v.W = P->W;
  v.Wb = P->Wb;
  v.block_term = (P->flags & SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT) ? 0 : 1;
  v.bt_lo = P->bt_lo;
  v.bt_hi = P->bt_hi;
  v.partial_bf16 = (P->flags & SPLITKV_FLAG_PARTIAL_BF16) ? 1 : 0;
  v.dynamic = dynamic ? 1 : 0;
  v.n_fwd_items = int(P->fwd_items.size());
  v.n_bwd_items = int(P->bwd_items.size());
  v.claim = reinterpret_cast<int*>(d + status_off + 128);   // after the two status words
  v.wait_limit_ns = P->wait_limit_ns;
  P->uploaded = true;
  return SPLITKV_OK;
}

int splitkv_plan_set_wait_limit(splitkv_plan_t* P, int64_t ns) {
  if (!P || ns < 0 || ns > kMaxWaitLimitNs) return SPLITKV_ERR_INVALID_ARG;
  P->wait_limit_ns = ns;
  P->dev.wait_limit_ns = ns;   // takes effect from the next launch (the device view is passed by value)
  return SPLITKV_OK;
}

int splitkv_plan_destroy(splitkv_plan_t* P) {
  if (!P) return SPLITKV_OK;
  int st = SPLITKV_OK;
  if (P->d_blob || P->upload_pending) {
    if (cudaDeviceSynchronize() != cudaSuccess) st = SPLITKV_ERR_CUDA;
  }
  if (P->d_blob) cudaFree(P->d_blob);
  if (P->h_pinned) cudaFreeHost(P->h_pinned);
  if (P->upload_ev) cudaEventDestroy(P->upload_ev);
  delete P;
  return st;
}

int splitkv_plan_stats(const splitkv_plan_t* P, splitkv_stats* out) {
  if (!P || !out) return SPLITKV_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  out->context_len = P->N;
  out->num_queries = P->Nq;
  out->num_chunks = P->num_chunks;
  out->num_entries = int32_t(P->entries.size());
  out->num_tiles = int32_t(P->tiles.size());
  out->num_fwd_items = int32_t(P->fwd_items.size());
  out->num_bwd_items = int32_t(P->bwd_items.size());
  out->num_workers = P->W;
  out->num_bwd_workers = P->Wb;
  uint64_t ctx = 0;
  for (uint64_t x : P->chunk_pairs) ctx += x;
  out->context_pairs = ctx * uint64_t(P->Hq);
  out->block_pairs = (P->flags & SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT)
                         ? 0
                         : uint64_t(P->Hq) * uint64_t(P->bt_hi - P->bt_lo) * uint64_t(P->bs) * uint64_t(P->bs);
  out->fwd_max_load = P->fwd_loads.empty() ? 0 : *std::max_element(P->fwd_loads.begin(), P->fwd_loads.end());
  out->bwd_max_load = P->bwd_loads.empty() ? 0 : *std::max_element(P->bwd_loads.begin(), P->bwd_loads.end());
  out->fwd_imbalance = imbalance(P->fwd_loads);
  out->bwd_imbalance = imbalance(P->bwd_loads);
  out->contig_imbalance = imbalance(P->contig_loads);
  out->plan_us = P->plan_us;
  return SPLITKV_OK;
}

int splitkv_plan_export(const splitkv_plan_t* P, int what, int64_t* out, int64_t capacity,
                        int64_t* count) {
  if (!P || !count || capacity < 0 || (capacity > 0 && !out)) return SPLITKV_ERR_INVALID_ARG;
  std::vector<int64_t> v;
  try {
    switch (what) {
      case SPLITKV_EXPORT_ENTRIES:
        for (const I4& e : P->entries) v.insert(v.end(), {int64_t(e.w), int64_t(e.x), int64_t(e.y), int64_t(e.z)});
        break;
      case SPLITKV_EXPORT_CHUNK_PAIRS:
        for (uint64_t x : P->chunk_pairs) v.push_back(int64_t(x));
        break;
      case SPLITKV_EXPORT_FWD_SCHEDULE:
      case SPLITKV_EXPORT_BWD_SCHEDULE: {
        const bool f = what == SPLITKV_EXPORT_FWD_SCHEDULE;
        const auto& items = f ? P->fwd_items : P->bwd_items;
        const auto& ptr = f ? P->fwd_worker_ptr : P->bwd_worker_ptr;
        const auto& order = f ? P->fwd_order : P->bwd_order;
        const int nw = f ? P->W : P->Wb;
        for (int w = 0; w < nw; ++w)
          for (int i = ptr[w]; i < ptr[w + 1]; ++i) {
            const Item& it = items[order[i]];
            v.insert(v.end(), {int64_t(w), int64_t(it.c), int64_t(it.g), int64_t(it.slice), int64_t(it.cost)});
          }
        break;
      }
      case SPLITKV_EXPORT_FWD_LOADS:
        for (uint64_t x : P->fwd_loads) v.push_back(int64_t(x));
        break;
      case SPLITKV_EXPORT_BWD_LOADS:
        for (uint64_t x : P->bwd_loads) v.push_back(int64_t(x));
        break;
      case SPLITKV_EXPORT_CONTIG_LOADS:
        for (uint64_t x : P->contig_loads) v.push_back(int64_t(x));
        break;
      case SPLITKV_EXPORT_FWD_LPT_ORDER:
      case SPLITKV_EXPORT_BWD_LPT_ORDER: {
        const bool f = what == SPLITKV_EXPORT_FWD_LPT_ORDER;
        const auto& items = f ? P->fwd_items : P->bwd_items;
        for (int32_t i : (f ? P->fwd_lpt : P->bwd_lpt)) {
          const Item& it = items[i];
          v.insert(v.end(), {int64_t(it.c), int64_t(it.g), int64_t(it.slice), int64_t(it.cost)});
        }
        break;
      }
      case SPLITKV_EXPORT_CHUNK_OWNER:
        for (int32_t r : P->chunk_owner) v.push_back(int64_t(r));
        break;
      case SPLITKV_EXPORT_QUERY_SHARD:
        v.insert(v.end(), {int64_t(P->rank), int64_t(P->R), int64_t(P->bt_lo), int64_t(P->bt_hi)});
        break;
      default:
        return SPLITKV_ERR_INVALID_ARG;
    }
  } catch (...) {
    return SPLITKV_ERR_NO_MEMORY;
  }
  *count = int64_t(v.size());
  if (capacity < *count) return out ? SPLITKV_ERR_WORKSPACE_TOO_SMALL : SPLITKV_OK;
  if (!v.empty()) std::memcpy(out, v.data(), v.size() * sizeof(int64_t));
  return SPLITKV_OK;
}

int splitkv_workspace_size(const splitkv_plan_t* P, int which, size_t* bytes) {
  if (!P || !bytes) return SPLITKV_ERR_INVALID_ARG;
  const long long E = (long long)P->entries.size();
  const size_t rb = (P->flags & SPLITKV_FLAG_PARTIAL_BF16) ? 2 : 4;
  if (which == SPLITKV_WS_FWD) {
    *bytes = splitkv::fwd_ws_layout(E, P->bs, P->Hq, P->d, rb).total;
  } else if (which == SPLITKV_WS_BWD) {
    *bytes = splitkv::bwd_ws_layout(E, int(P->Nq), P->bs, P->Hq, P->d, rb).total;
  } else {
    return SPLITKV_ERR_INVALID_ARG;
  }
  return SPLITKV_OK;
}

}  // extern "C"

// Accessors for the attention entry points (api.cu).
namespace splitkv {
const DevPlan* plan_device_view(const splitkv_plan_t* P) { return P->uploaded ? &P->dev : nullptr; }
void plan_ranks(const splitkv_plan_t* P, int* R, int* rank) {
  *R = P->R;
  *rank = P->rank;
}
}  // namespace splitkv
