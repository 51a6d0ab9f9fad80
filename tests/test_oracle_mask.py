"""Pins of the oracle's mask structure (CPU only).

Rule: "Split-KV speeds diffusion drafter training..." news page, section "Why
short queries change the problem" (each block attends to the preceding context
of its own sample and to all tokens inside the block) and section "Balance
actual attention work" (chunk cost = actual attention usage).
"""

import json
import os

import numpy as np
import pytest

from oracle import mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _random_problem(rng, max_samples=4, max_len=40, max_anchors=6):
    S = int(rng.integers(1, max_samples + 1))
    lens = rng.integers(1, max_len + 1, size=S).astype(np.int32)
    N = int(lens.sum())
    A = int(rng.integers(1, max_anchors + 1))
    anchors = np.sort(rng.choice(N, size=min(A, N), replace=False)).astype(np.int32)
    return lens, anchors


def _token_sample_brute(lens):
    """Sample id of every packed token, by walking the tokens one by one."""
    out = []
    for s, L in enumerate(lens):
        out.extend([s] * int(L))
    return out


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "mask_hand.json")))
    lens, anchors = g["sample_lens"], g["anchors"]
    assert mask.sample_starts(lens) == g["starts"]
    assert mask.anchor_sample(lens, anchors) == g["anchor_sample"]
    assert [list(x) for x in mask.context_interval(lens, anchors)] == g["intervals"]
    assert [list(x) for x in mask.chunk_entries(lens, anchors, g["kv_chunk"])] == g["entries"]
    assert mask.chunk_pairs(lens, anchors, g["block_size"], g["kv_chunk"]).tolist() == g["chunk_pairs"]
    assert mask.chunk_pairs_loops(lens, anchors, g["block_size"], g["kv_chunk"]) == g["chunk_pairs"]


@pytest.mark.parametrize("seed", range(20))
def test_intervals_match_token_level_rule(seed):
    """Allowed context keys of a block = tokens of the anchor's sample strictly before the anchor."""
    rng = np.random.default_rng(seed)
    lens, anchors = _random_problem(rng)
    tok_sample = _token_sample_brute(lens)
    for (lo, hi), a in zip(mask.context_interval(lens, anchors), anchors):
        brute = [j for j in range(len(tok_sample)) if tok_sample[j] == tok_sample[a] and j < a]
        assert list(range(lo, hi)) == brute


@pytest.mark.parametrize("seed", range(20))
def test_chunk_entries_and_pairs_brute(seed):
    rng = np.random.default_rng(100 + seed)
    lens, anchors = _random_problem(rng)
    C = int(rng.integers(1, 17))
    bs = int(rng.integers(1, 5))
    tok_sample = _token_sample_brute(lens)
    N = len(tok_sample)
    # entries: every (chunk, block) whose allowed key set meets the chunk, with exact key range
    want = []
    for c in range((N + C - 1) // C):
        for b, a in enumerate(anchors):
            keys = [j for j in range(c * C, min((c + 1) * C, N))
                    if tok_sample[j] == tok_sample[a] and j < a]
            if keys:
                assert keys == list(range(keys[0], keys[-1] + 1))   # contiguous
                want.append((c, b, keys[0], keys[-1] + 1))
    assert mask.chunk_entries(lens, anchors, C) == want
    pairs = mask.chunk_pairs(lens, anchors, bs, C)
    assert pairs.tolist() == mask.chunk_pairs_loops(lens, anchors, bs, C)
    # closed form: sum_c pairs_c = bs * sum_b (a_b - S_{s(b)})
    starts = mask.sample_starts(lens)
    closed = bs * sum(int(a) - starts[tok_sample[a]] for a in anchors)
    assert int(pairs.sum()) == closed


def test_anchor_at_sample_start_has_empty_context():
    lens = [4, 4]
    anchors = [0, 4]
    assert mask.context_interval(lens, anchors) == [(0, 0), (4, 4)]
    assert mask.chunk_entries(lens, anchors, 2) == []
    assert mask.chunk_pairs(lens, anchors, 16, 2).tolist() == [0, 0, 0, 0]


def test_anchor_outside_context_rejected():
    with pytest.raises(ValueError):
        mask.anchor_sample([3, 2], [5])


def test_chunk_straddling_samples():
    # chunk [4, 8) straddles samples [0,6) and [6,10): serves blocks of both
    lens, anchors = [6, 4], [5, 9]
    ent = mask.chunk_entries(lens, anchors, 4)
    assert ent == [(0, 0, 0, 4), (1, 0, 4, 5), (1, 1, 6, 8), (2, 1, 8, 9)]
