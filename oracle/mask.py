"""Mask structure of anchor-block attention (fp64 oracle; test infrastructure).

[news] "Why short queries change the problem": anchors open blocks of draft
tokens; each block attends to the preceding context within its own sample and
to all tokens inside the block.  Samples are packed back to back into one
context (sample s occupies [S_s, S_s + L_s)).

Where the block's own tokens live is not fixed by the pages.  Reading A (the
default): they are the draft block's own keys and values, separate from the
context, so a block's context interval ends at its anchor.  Reading B
(`block_keys_in_context`): they are the context positions after the anchor, so
the interval runs on to min(a_b + bs, end of the sample) and the block has no
keys besides the context.

[news] "Balance actual attention work": the context is cut into chunks and a
chunk's cost is its actual attention usage, i.e. the number of allowed
(query, key) pairs that fall into it.  Chunks are fixed-length pieces of the
packed context, [c*C, min((c+1)*C, N)), regardless of sample boundaries.
"""

from __future__ import annotations

from typing import List, Tuple

import numpy as np


def sample_starts(sample_lens) -> List[int]:
    """S_s: packed start offset of every sample."""
    starts = []
    acc = 0
    for L in sample_lens:
        starts.append(acc)
        acc += int(L)
    return starts


def anchor_sample(sample_lens, anchors) -> List[int]:
    """s(b): the sample holding anchor a_b, i.e. S_s <= a_b < S_s + L_s."""
    starts = sample_starts(sample_lens)
    out = []
    for a in anchors:
        a = int(a)
        found = -1
        for s, (S, L) in enumerate(zip(starts, sample_lens)):
            if S <= a < S + int(L):
                found = s
                break
        if found < 0:
            raise ValueError(f"anchor {a} lies outside the packed context")
        out.append(found)
    return out


def context_interval(sample_lens, anchors, block_size: int = 0,
                     block_keys_in_context: bool = False) -> List[Tuple[int, int]]:
    """Allowed context keys of block b: [S_{s(b)}, a_b) (preceding context of its own sample);
    under reading B, [S_{s(b)}, min(a_b + bs, S_{s(b)} + L_{s(b)}))."""
    starts = sample_starts(sample_lens)
    out = []
    for s, a in zip(anchor_sample(sample_lens, anchors), anchors):
        end = int(a)
        if block_keys_in_context:
            end = min(int(a) + int(block_size), starts[s] + int(sample_lens[s]))
        out.append((starts[s], end))
    return out


def num_chunks(context_len: int, kv_chunk: int) -> int:
    return (int(context_len) + kv_chunk - 1) // kv_chunk


def chunk_entries(sample_lens, anchors, kv_chunk: int, block_size: int = 0,
                  block_keys_in_context: bool = False) -> List[Tuple[int, int, int, int]]:
    """Every (chunk c, block b, lo, hi) whose clipped interval [lo, hi) is non-empty.

    lo = max(S_s, c*C), hi = min(e_b, (c+1)*C, N), with e_b the interval end
    (a_b, or the reading-B end).  Ordered by chunk, then block.
    """
    N = int(np.sum(sample_lens))
    iv = context_interval(sample_lens, anchors, block_size, block_keys_in_context)
    out = []
    for c in range(num_chunks(N, kv_chunk)):
        c0, c1 = c * kv_chunk, min((c + 1) * kv_chunk, N)
        for b, (S, a) in enumerate(iv):
            lo, hi = max(S, c0), min(a, c1)
            if lo < hi:
                out.append((c, b, lo, hi))
    return out


def chunk_pairs(sample_lens, anchors, block_size: int, kv_chunk: int,
                block_keys_in_context: bool = False) -> np.ndarray:
    """pairs_c: allowed (query row, context key) pairs inside each chunk, per query head.

    Evaluated straight from the definition: for every block, mark the context
    keys it may read, count the marks that fall into each chunk, and multiply
    by the block's bs query rows.  (Under reading A the in-block keys are not
    context keys and belong to no chunk.)
    """
    N = int(np.sum(sample_lens))
    nc = num_chunks(N, kv_chunk)
    counts = np.zeros(nc, dtype=np.int64)
    keys = np.arange(N, dtype=np.int64)
    chunk_of_key = keys // kv_chunk
    for S, a in context_interval(sample_lens, anchors, block_size, block_keys_in_context):
        allowed = (keys >= S) & (keys < a)
        counts += np.bincount(chunk_of_key[allowed], minlength=nc).astype(np.int64)
    return counts * int(block_size)


def chunk_pairs_loops(sample_lens, anchors, block_size: int, kv_chunk: int,
                      block_keys_in_context: bool = False) -> List[int]:
    """Same count as chunk_pairs by a plain triple loop (chunks x blocks x keys); small inputs only."""
    N = int(np.sum(sample_lens))
    iv = context_interval(sample_lens, anchors, block_size, block_keys_in_context)
    out = []
    for c in range(num_chunks(N, kv_chunk)):
        total = 0
        for (S, a) in iv:
            for j in range(c * kv_chunk, min((c + 1) * kv_chunk, N)):
                if S <= j < a:
                    total += block_size
        out.append(total)
    return out
