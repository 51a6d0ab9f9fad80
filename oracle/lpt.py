"""Cost-aware LPT planning of KV chunks onto workers (oracle; test infrastructure).

[news] "Balance actual attention work": each context chunk gets a cost equal to
its actual attention usage; LPT sorts chunks by cost and hands the expensive
ones first to the least-loaded eligible worker, keeping chunk counts equal
(device mode).  [digest] Abstract: "cost-aware longest-processing-time-first".

Readings where the pages are silent (integer arithmetic, so bit-exact):

* work item = (chunk c, KV head g[, slice]); cost = realised pairs served by the
  item = G * pairs_c (G query heads read KV head g), or G * bs * sum(hi - lo)
  over the blocks of a slice;
* slicing: the chunk's entries are ordered by (lo, hi, b) and cut into query
  tiles of rows_per_tile // (G * bs) blocks; consecutive groups of q_slice tiles
  form the slices of the item;
* items are ordered by cost descending, ties by (c, g, slice) ascending;
* each goes to the eligible worker of minimum load, ties to the lowest id;
* zero-cost items are dropped;
* equal-count mode, n items on W workers, n = q W + r: a worker is eligible
  while it holds fewer than q items, or holds q and fewer than r workers hold
  q + 1;
* imbalance = max load / mean load - 1 over all W workers;
* the "unbalanced" baseline keeps chunks in contiguous order: the n_chunks * Hkv
  unsliced items in (c, g) order, item i to worker floor(i W / n).

Optional tile cost of the backward schedule (this library's refinement for its
dK/dV kernel, not the pages' rule): the cost of a (chunk, head) item is the work
that kernel executes, in (row, key) pairs of whole tiles -- rows_per_tile-row
query tiles against key_tile-key key tiles -- so that partly filled tiles count
as full ones: for every key tile [k0, k0 + key_tile) of the chunk, k0 = cC,
cC + key_tile, ..., below min((c+1)C, N), one step per query tile whose key
range meets it; cost = steps * rows_per_tile * key_tile.

Optional tile cost of the forward schedule (the same refinement for the forward
kernel): a forward item's query tiles are taken two at a time from its first
tile, and each pair runs over the key tiles of its joint key range [min lo,
max hi), starting at min lo; a pair costs 2 * ceil((max hi - min lo) / key_tile)
steps (a last single tile, 1 * ceil((hi - lo) / key_tile)); cost = steps *
rows_per_tile * key_tile.
"""

from __future__ import annotations

from typing import Dict, List, Tuple

from .mask import chunk_entries, chunk_pairs, num_chunks


def query_tiles(sample_lens, anchors, block_size: int, kv_chunk: int, G: int, rows_per_tile: int = 128,
                block_keys_in_context: bool = False) -> Dict[int, List[Tuple[int, int]]]:
    """Per chunk, its query tiles' key ranges [min lo, max hi): consecutive groups of
    rows_per_tile // (G * bs) entries in (lo, hi, block) order."""
    bs = int(block_size)
    bpt = rows_per_tile // (G * bs)
    per_chunk: Dict[int, list] = {}
    for (c, b, lo, hi) in chunk_entries(sample_lens, anchors, kv_chunk, bs, block_keys_in_context):
        per_chunk.setdefault(c, []).append((lo, hi, b))
    out = {}
    for c in sorted(per_chunk):
        ents = sorted(per_chunk[c])
        out[c] = [(min(e[0] for e in ents[i:i + bpt]), max(e[1] for e in ents[i:i + bpt]))
                  for i in range(0, len(ents), bpt)]
    return out


def bwd_tile_cost(tiles, c: int, kv_chunk: int, context_len: int, rows_per_tile: int = 128,
                  key_tile: int = 128) -> int:
    """Executed (row, key) pairs of the dK/dV kernel on chunk c: per key tile of the chunk,
    one step per query tile meeting it."""
    steps = 0
    for k0 in range(c * kv_chunk, min((c + 1) * kv_chunk, context_len), key_tile):
        steps += sum(1 for (lo, hi) in tiles if lo < k0 + key_tile and hi > k0)
    return steps * rows_per_tile * key_tile


def forward_tile_cost(tiles, rows_per_tile: int = 128, key_tile: int = 128) -> int:
    """Executed (row, key) pairs of the forward kernel on one item's query tiles (their
    key ranges, in item order): the tiles go in twos, each two over their joint key range."""
    steps = 0
    for i in range(0, len(tiles), 2):
        two = tiles[i:i + 2]
        lo = min(t[0] for t in two)
        hi = max(t[1] for t in two)
        n_key_tiles = -(-(hi - lo) // key_tile)
        steps += len(two) * n_key_tiles
    return steps * rows_per_tile * key_tile


def work_items(sample_lens, anchors, block_size: int, kv_chunk: int, num_q_heads: int,
               num_kv_heads: int, q_slice: int = 0, rows_per_tile: int = 128,
               block_keys_in_context: bool = False, tile_cost: bool = False,
               fwd_tile_cost: bool = False) -> List[Tuple[Tuple[int, int, int], int]]:
    """All work items ((c, g, slice), cost), zero-cost ones included.  tile_cost: whole-chunk
    items of the backward schedule costed by the dK/dV kernel's executed tile work;
    fwd_tile_cost: items of the forward schedule (sliced or not) costed by the forward
    kernel's executed tile work."""
    G = num_q_heads // num_kv_heads
    bs = int(block_size)
    items = []
    if fwd_tile_cost:
        if tile_cost:
            raise ValueError("tile_cost and fwd_tile_cost describe different schedules")
        N = int(sum(int(L) for L in sample_lens))
        tiles = query_tiles(sample_lens, anchors, bs, kv_chunk, G, rows_per_tile, block_keys_in_context)
        for c in range(num_chunks(N, kv_chunk)):
            ts = tiles.get(c, [])
            if q_slice <= 0:
                groups = [ts]
            else:
                groups = [ts[i:i + q_slice] for i in range(0, len(ts), q_slice)]
            for s, grp in enumerate(groups):
                cost = forward_tile_cost(grp, rows_per_tile)
                for g in range(num_kv_heads):
                    items.append(((c, g, s), int(cost)))
        return items
    if tile_cost:
        if q_slice > 0:
            raise ValueError("the tile cost applies to the backward schedule (whole chunks)")
        N = int(sum(int(L) for L in sample_lens))
        tiles = query_tiles(sample_lens, anchors, bs, kv_chunk, G, rows_per_tile, block_keys_in_context)
        for c in range(num_chunks(N, kv_chunk)):
            cost = bwd_tile_cost(tiles.get(c, []), c, kv_chunk, N, rows_per_tile)
            for g in range(num_kv_heads):
                items.append(((c, g, 0), int(cost)))
        return items
    if q_slice <= 0:
        pairs = chunk_pairs(sample_lens, anchors, bs, kv_chunk, block_keys_in_context)
        for c, p in enumerate(pairs):
            for g in range(num_kv_heads):
                items.append(((c, g, 0), int(G * p)))
        return items
    blocks_per_tile = rows_per_tile // (G * bs)
    per_chunk: Dict[int, list] = {}
    for (c, b, lo, hi) in chunk_entries(sample_lens, anchors, kv_chunk, bs, block_keys_in_context):
        per_chunk.setdefault(c, []).append((lo, hi, b))
    for c in sorted(per_chunk):
        ents = sorted(per_chunk[c])
        per_slice = blocks_per_tile * q_slice
        for s0 in range(0, len(ents), per_slice):
            cost = G * bs * sum(hi - lo for (lo, hi, _) in ents[s0:s0 + per_slice])
            for g in range(num_kv_heads):
                items.append(((c, g, s0 // per_slice), int(cost)))
    return items


def lpt_order(items):
    """The order in which LPT hands out items: positive-cost items by cost descending,
    ties by key ascending."""
    live = [(key, cost) for (key, cost) in items if cost > 0]
    live.sort(key=lambda it: (-it[1], it[0]))
    return live


def lpt(items, num_workers: int, equal_count: bool = False):
    """Assign items to workers longest-first; returns (lists, loads).

    lists[w] holds the item keys of worker w in assignment order.
    """
    live = lpt_order(items)
    W = int(num_workers)
    n = len(live)
    q, r = divmod(n, W)
    loads = [0] * W
    counts = [0] * W
    lists: List[list] = [[] for _ in range(W)]
    for key, cost in live:
        n_full = sum(1 for x in counts if x == q + 1)
        best = -1
        for w in range(W):
            if equal_count:
                ok = counts[w] < q or (counts[w] == q and n_full < r)
            else:
                ok = True
            if ok and (best < 0 or loads[w] < loads[best]):
                best = w
        loads[best] += cost
        counts[best] += 1
        lists[best].append(key)
    return lists, loads


def contiguous(items, num_workers: int):
    """Chunks left in contiguous order: item i of n (c, g order) -> worker floor(i W / n)."""
    ordered = sorted(items, key=lambda it: it[0])
    W = int(num_workers)
    n = len(ordered)
    loads = [0] * W
    lists: List[list] = [[] for _ in range(W)]
    for i, (key, cost) in enumerate(ordered):
        w = (i * W) // n
        loads[w] += cost
        lists[w].append(key)
    return lists, loads


def imbalance(loads) -> float:
    """max load / mean load - 1 (0 for an all-zero load vector)."""
    total = sum(loads)
    if total == 0:
        return 0.0
    mean = total / len(loads)
    return max(loads) / mean - 1.0


def makespan(loads) -> int:
    return max(loads) if loads else 0
