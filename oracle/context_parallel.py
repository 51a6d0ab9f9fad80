"""Split-KV over several ranks, by definition, in float64 (oracle; test infrastructure).

[news] "Exchange the smaller side": every device keeps its own share of the
long context's keys and values; the short query side (the draft blocks) is
exchanged instead, each device computes partial attention of all queries
against its keys, and the partials are combined exactly with their
normalisation statistics.  [news] "Balance actual attention work": the chunks
go to devices by cost-aware LPT with equal chunk counts (the device rule).

Readings where the pages are silent:

* ownership: whole chunks, every chunk (zero-cost ones included: each chunk's
  keys and values live somewhere, and equal counts are about memory); chunk
  cost = Hq * pairs_c, the chunk's realised (row, key) pairs over all query
  heads; LPT order = cost descending, ties by chunk ascending; each chunk to the
  eligible rank of least load, ties to the lowest rank; with n = q R + r chunks
  a rank is eligible while it holds fewer than q, or q while fewer than r ranks
  hold q + 1;
* the "unbalanced" baseline the pages compare against keeps chunks in order: chunk c
  to rank floor(c R / n);
* query side: blocks are split into R contiguous ranges, rank r owning
  [floor(r A / R), floor((r + 1) A / R)); the owner of a block holds its draft
  keys/values (kb, vb) and adds the in-block term;
* a rank's result for a query row is the exact partial over its keys: (O_r,
  LSE_r) with O_r the softmax-weighted mean over the rank's allowed keys and
  LSE_r their log-sum-exp (O_r = 0, LSE_r = -inf when the rank holds none);
* combine: O = sum_r exp(LSE_r - LSE) O_r with LSE = log sum_r exp(LSE_r);
* backward with the final O, LSE (so P_ij = exp(s_ij - LSE_i) is the true
  probability): every rank forms, over its own keys, dQ_r = scale sum_j dS_ij
  k_j with dS = P (dP - Delta), Delta = rowsum(dout * O); dQ = sum_r dQ_r; the
  gradients of a rank's context keys (and of its blocks' draft keys) are
  complete on that rank.
"""

from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

from .attention import NEG_INF, merge, partial
from .mask import chunk_pairs, context_interval


def chunk_owners(sample_lens, anchors, block_size: int, kv_chunk: int, num_q_heads: int, num_ranks: int,
                 block_keys_in_context: bool = False) -> List[int]:
    """Owning rank of every chunk (equal-count LPT over all chunks, cost Hq * pairs_c)."""
    pairs = chunk_pairs(sample_lens, anchors, block_size, kv_chunk, block_keys_in_context)
    n = len(pairs)
    R = int(num_ranks)
    q, r = divmod(n, R)
    order = sorted(range(n), key=lambda c: (-int(num_q_heads) * int(pairs[c]), c))
    loads = [0] * R
    counts = [0] * R
    owner = [-1] * n
    for c in order:
        n_full = sum(1 for x in counts if x == q + 1)
        best = -1
        for w in range(R):
            ok = counts[w] < q or (counts[w] == q and n_full < r)
            if ok and (best < 0 or loads[w] < loads[best]):
                best = w
        loads[best] += int(num_q_heads) * int(pairs[c])
        counts[best] += 1
        owner[c] = best
    return owner


def chunk_owners_contiguous(num_chunks: int, num_ranks: int) -> List[int]:
    """The "unbalanced" device baseline ([news] "Balance actual attention work"): chunks left
    in order, chunk c to rank floor(c R / n) -- equal counts, whatever their costs."""
    return [(c * int(num_ranks)) // int(num_chunks) for c in range(int(num_chunks))]


def query_shard(num_blocks: int, num_ranks: int, rank: int) -> Tuple[int, int]:
    """Blocks [lo, hi) whose queries, draft keys and in-block term rank `rank` holds."""
    return (rank * num_blocks) // num_ranks, ((rank + 1) * num_blocks) // num_ranks


def _rank_keys(k, v, kb, vb, S, a, b, bs, g, kv_chunk, owned, own_block, in_context):
    """Keys (and values) of block b, KV head g that the rank holds, and their positions
    (context index, or -1 - t for draft key t)."""
    keys, vals, pos = [], [], []
    for j in range(S, a):
        if owned[j // kv_chunk]:
            keys.append(k[j, g]); vals.append(v[j, g]); pos.append(j)
    if not in_context and own_block:
        for t in range(bs):
            keys.append(kb[b * bs + t, g]); vals.append(vb[b * bs + t, g]); pos.append(-1 - t)
    d = k.shape[2]
    if not keys:
        return np.zeros((0, d)), np.zeros((0, d)), []
    return np.array(keys), np.array(vals), pos


def rank_fwd(q, k, v, kb, vb, sample_lens, anchors, block_size: int, kv_chunk: int, scale: float,
             owner: Sequence[int], rank: int, num_ranks: int, block_keys_in_context: bool = False):
    """(O_r [Nq, Hq, d], LSE_r [Nq, Hq]) of rank `rank`: exact attention of every query row
    over the keys the rank holds."""
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    bs = int(block_size)
    owned = [o == rank for o in owner]
    b_lo, b_hi = query_shard(len(anchors), num_ranks, rank)
    O = np.zeros((Nq, Hq, d))
    LSE = np.full((Nq, Hq), NEG_INF)
    for b, (S, a) in enumerate(context_interval(sample_lens, anchors, bs, block_keys_in_context)):
        rows = slice(b * bs, (b + 1) * bs)
        for h in range(Hq):
            keys, vals, _ = _rank_keys(k, v, kb, vb, S, a, b, bs, h // G, kv_chunk, owned,
                                       b_lo <= b < b_hi, block_keys_in_context)
            m, l, o = partial(scale * (q[rows, h, :] @ keys.T), vals)
            live = l > 0
            O[rows, h, :] = o
            LSE[rows, h] = np.where(live, m + np.log(np.where(live, l, 1.0)), NEG_INF)
    return O, LSE


def combine_ranks(O_parts: np.ndarray, LSE_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Exact combine of the ranks' results: O_parts [R, ..., d], LSE_parts [R, ...].  A
    normalised partial with log-sum-exp LSE_r is the record (m, l) = (LSE_r, 1)."""
    R = O_parts.shape[0]
    shape = LSE_parts.shape[1:]
    d = O_parts.shape[-1]
    recs = []
    for r in range(R):
        lse = LSE_parts[r].reshape(-1)
        live = np.isfinite(lse)
        recs.append((np.where(live, lse, NEG_INF), live.astype(np.float64), O_parts[r].reshape(-1, d)))
    o, lse = merge(recs)
    return o.reshape(shape + (d,)), lse.reshape(shape)


def rank_bwd(q, k, v, kb, vb, dout, o, lse, sample_lens, anchors, block_size: int, kv_chunk: int,
             scale: float, owner: Sequence[int], rank: int, num_ranks: int,
             block_keys_in_context: bool = False) -> Dict[str, np.ndarray]:
    """Rank `rank`'s backward over its keys, given the final o, lse: dq (its share, all
    rows), dk / dv (non-zero only on its chunks), dkb / dvb (non-zero only on its blocks)."""
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    bs = int(block_size)
    owned = [x == rank for x in owner]
    b_lo, b_hi = query_shard(len(anchors), num_ranks, rank)
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dkb": None if block_keys_in_context else np.zeros_like(kb),
           "dvb": None if block_keys_in_context else np.zeros_like(vb)}
    delta = (dout * o).sum(axis=2)                     # [Nq, Hq]
    for b, (S, a) in enumerate(context_interval(sample_lens, anchors, bs, block_keys_in_context)):
        rows = slice(b * bs, (b + 1) * bs)
        for h in range(Hq):
            g = h // G
            keys, vals, pos = _rank_keys(k, v, kb, vb, S, a, b, bs, g, kv_chunk, owned,
                                         b_lo <= b < b_hi, block_keys_in_context)
            if not pos:
                continue
            P = np.exp(scale * (q[rows, h, :] @ keys.T) - lse[rows, h][:, None])
            dP = dout[rows, h, :] @ vals.T
            dS = P * (dP - delta[rows, h][:, None])
            out["dq"][rows, h, :] += scale * (dS @ keys)
            dkeys = scale * (dS.T @ q[rows, h, :])
            dvals = P.T @ dout[rows, h, :]
            for i, j in enumerate(pos):
                if j >= 0:
                    out["dk"][j, g] += dkeys[i]
                    out["dv"][j, g] += dvals[i]
                else:
                    out["dkb"][b * bs + (-1 - j), g] += dkeys[i]
                    out["dvb"][b * bs + (-1 - j), g] += dvals[i]
    return out
