"""Pins of the oracle's LPT planner (CPU only).

LPT as stated on the news page, section "Balance actual attention work", and
in the digest Abstract.  Pins: hand-worked assignments, Graham's makespan bound
(4/3 - 1/(3m)) against an exhaustive optimum, the equal-count rule against an
exhaustive equal-count optimum, and the cost bookkeeping.
"""

import itertools
import json
import os

import numpy as np
import pytest

from oracle import lpt, mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _items(costs):
    return [((i, 0, 0), int(c)) for i, c in enumerate(costs)]


def test_hand_worked_cases():
    g = json.load(open(os.path.join(GOLDEN, "lpt_hand.json")))
    for case in g["cases"]:
        lists, loads = lpt.lpt(_items(case["costs"]), case["workers"], case["equal_count"])
        assert [[k[0] for k in l] for l in lists] == case["lists"], case["_worked"]
        assert loads == case["loads"]


def _opt(costs, m, equal_count=False):
    n = len(costs)
    best = None
    q, r = divmod(n, m)
    for assign in itertools.product(range(m), repeat=n):
        if equal_count:
            cnt = np.bincount(assign, minlength=m)
            if sorted(cnt.tolist()) != sorted([q + 1] * r + [q] * (m - r)):
                continue
        loads = [0] * m
        for c, w in zip(costs, assign):
            loads[w] += c
        ms = max(loads)
        best = ms if best is None else min(best, ms)
    return best


@pytest.mark.parametrize("seed", range(40))
def test_graham_bound_vs_exhaustive(seed):
    rng = np.random.default_rng(seed)
    m = int(rng.integers(2, 5))
    n = int(rng.integers(m + 1, 9))
    costs = rng.integers(1, 50, size=n).tolist()
    _, loads = lpt.lpt(_items(costs), m)
    opt = _opt(costs, m)
    assert max(loads) <= (4.0 / 3.0 - 1.0 / (3 * m)) * opt + 1e-9


@pytest.mark.parametrize("seed", range(40))
def test_equal_count_counts_and_bound(seed):
    """Counts differ by at most one; makespan within 4/3 - 1/(3m) of the equal-count optimum
    on these instances (the bound observed; the pages state only that counts stay equal)."""
    rng = np.random.default_rng(1000 + seed)
    m = int(rng.integers(2, 4))
    n = int(rng.integers(m + 1, 9))
    costs = rng.integers(1, 50, size=n).tolist()
    lists, loads = lpt.lpt(_items(costs), m, equal_count=True)
    cnt = sorted(len(l) for l in lists)
    q, r = divmod(n, m)
    assert cnt == sorted([q + 1] * r + [q] * (m - r))
    opt = _opt(costs, m, equal_count=True)
    assert max(loads) <= (4.0 / 3.0 - 1.0 / (3 * m)) * opt + 1e-9


def test_every_item_assigned_once_and_order_is_longest_first():
    rng = np.random.default_rng(3)
    costs = rng.integers(0, 100, size=60).tolist()
    lists, loads = lpt.lpt(_items(costs), 7)
    got = sorted(k[0] for l in lists for k in l)
    assert got == [i for i, c in enumerate(costs) if c > 0]
    for l in lists:
        cs = [costs[k[0]] for k in l]
        assert cs == sorted(cs, reverse=True)
    assert loads == [sum(costs[k[0]] for k in l) for l in lists]


def test_imbalance_definition():
    assert lpt.imbalance([10, 10, 10]) == 0.0
    assert abs(lpt.imbalance([12, 6, 6]) - (12 / 8 - 1)) < 1e-15
    assert lpt.imbalance([0, 0]) == 0.0


def test_contiguous_baseline_equal_lengths():
    items = _items([5, 0, 3, 9, 1, 1, 2])
    lists, loads = lpt.contiguous(items, 3)
    # floor(i*3/7): i=0,1,2 -> 0; 3,4 -> 1; 5,6 -> 2
    assert [[k[0] for k in l] for l in lists] == [[0, 1, 2], [3, 4], [5, 6]]
    assert loads == [8, 10, 3]


@pytest.mark.parametrize("q_slice", [0, 1, 2])
def test_item_costs_sum_to_realised_pairs(q_slice):
    rng = np.random.default_rng(11)
    lens = rng.integers(20, 200, size=5).astype(np.int32)
    N = int(lens.sum())
    anchors = np.sort(rng.choice(N, size=24, replace=False)).astype(np.int32)
    bs, C, Hq, Hkv = 4, 64, 8, 2
    items = lpt.work_items(lens, anchors, bs, C, Hq, Hkv, q_slice=q_slice, rows_per_tile=32)
    pairs = mask.chunk_pairs(lens, anchors, bs, C)
    total = sum(c for _, c in items)
    assert total == Hq * int(pairs.sum())
    per_chunk = {}
    for (c, g, s), cost in items:
        per_chunk[c] = per_chunk.get(c, 0) + cost
    for c, p in enumerate(pairs):
        assert per_chunk.get(c, 0) == Hq * int(p)


# ---------------------------------------------------------------------------
# optional tile cost (executed tile work)
# ---------------------------------------------------------------------------

def test_tile_cost_hand_worked():
    # one sample of 300 tokens, bs 16, G 1, 2-block (32-row) tiles, chunks of 128 keys
    lens, anchors, bs, C = [300], [50, 60, 200, 250], 16, 128
    tiles = lpt.query_tiles(lens, anchors, bs, C, 1, rows_per_tile=32)
    # chunk 0 entries (0,50),(0,60),(0,128),(0,128) -> tiles [0,60), [0,128); chunk 1: [128,250)
    assert tiles == {0: [(0, 60), (0, 128)], 1: [(128, 250)]}
    assert lpt.bwd_tile_cost(tiles[0], 0, C, 300, 32) == 2 * 32 * 128   # key tile [0,128): both tiles
    assert lpt.bwd_tile_cost(tiles[1], 1, C, 300, 32) == 1 * 32 * 128
    items = dict(lpt.work_items(lens, anchors, bs, C, 1, 1, rows_per_tile=32, tile_cost=True))
    assert items == {(0, 0, 0): 8192, (1, 0, 0): 4096, (2, 0, 0): 0}
    # the pages' pair cost of the same chunks: bs * sum(hi - lo)
    pairs = dict(lpt.work_items(lens, anchors, bs, C, 1, 1))
    assert pairs == {(0, 0, 0): 16 * (50 + 60 + 128 + 128), (1, 0, 0): 16 * (72 + 122), (2, 0, 0): 0}


@pytest.mark.parametrize("seed", range(12))
def test_tile_cost_bounds_pair_cost(seed):
    """Executed tile work covers every allowed pair: per item it is at least the pair cost."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 400, size=rng.integers(1, 5)).tolist()
    N = sum(lens)
    heads = [(1, 1), (4, 1), (8, 2)][seed % 3]
    bs = [4, 8, 16][seed % 3]
    anchors = rng.integers(0, N, size=rng.integers(1, 30)).tolist()
    C = int(rng.integers(16, 300))
    tc = dict(lpt.work_items(lens, anchors, bs, C, heads[0], heads[1], tile_cost=True))
    pc = dict(lpt.work_items(lens, anchors, bs, C, heads[0], heads[1]))
    assert set(pc) == set(tc)
    for key, cost in pc.items():
        assert tc[key] >= cost, key


def test_tile_cost_equals_pair_cost_for_full_aligned_tiles():
    # one block per 128-row tile (G * bs = 128) and every interval a whole number of key tiles
    lens, bs, C = [1024], 16, 256
    anchors = [512, 512, 768, 768]
    tc = dict(lpt.work_items(lens, anchors, bs, C, 8, 1, tile_cost=True))
    pc = dict(lpt.work_items(lens, anchors, bs, C, 8, 1))
    assert tc == pc


# ---------------------------------------------------------------------------
# optional tile cost of the forward schedule (tiles in twos over their joint key range)
# ---------------------------------------------------------------------------

def test_forward_tile_cost_hand_worked():
    # samples [0, 300) and [300, 600); bs 16, G 1, 2-block (32-row) tiles, one 512-key chunk in use
    lens, anchors, bs, C = [300, 300], [50, 60, 400, 410], 16, 512
    tiles = lpt.query_tiles(lens, anchors, bs, C, 1, rows_per_tile=32)
    # entries (0,50), (0,60), (300,400), (300,410) -> tiles [0,60), [300,410)
    assert tiles == {0: [(0, 60), (300, 410)]}
    # together they run over [0, 410): 4 key tiles each -> 8 steps
    assert lpt.forward_tile_cost(tiles[0], 32) == 8 * 32 * 128
    # alone: [0, 60) one key tile; [300, 410) one key tile starting at 300
    assert lpt.forward_tile_cost(tiles[0][:1], 32) == 32 * 128
    assert lpt.forward_tile_cost(tiles[0][1:], 32) == 32 * 128
    whole = dict(lpt.work_items(lens, anchors, bs, C, 1, 1, rows_per_tile=32, fwd_tile_cost=True))
    assert whole == {(0, 0, 0): 8 * 4096, (1, 0, 0): 0}
    sliced = dict(lpt.work_items(lens, anchors, bs, C, 1, 1, q_slice=1, rows_per_tile=32, fwd_tile_cost=True))
    assert sliced == {(0, 0, 0): 4096, (0, 0, 1): 4096}
    # the pages' pair cost of the chunk: bs * sum(hi - lo)
    assert dict(lpt.work_items(lens, anchors, bs, C, 1, 1)) == {(0, 0, 0): 16 * (50 + 60 + 100 + 110), (1, 0, 0): 0}
    with pytest.raises(ValueError):
        lpt.work_items(lens, anchors, bs, C, 1, 1, tile_cost=True, fwd_tile_cost=True)


@pytest.mark.parametrize("seed", range(12))
def test_forward_tile_cost_bounds_pair_cost(seed):
    """Executed tile work covers every allowed pair, sliced or not."""
    rng = np.random.default_rng(50 + seed)
    lens = rng.integers(1, 400, size=rng.integers(1, 5)).tolist()
    N = sum(lens)
    heads = [(1, 1), (4, 1), (8, 2)][seed % 3]
    bs = [4, 8, 16][seed % 3]
    anchors = rng.integers(0, N, size=rng.integers(1, 30)).tolist()
    C = int(rng.integers(16, 300))
    for q_slice in (0, 1, 2, 3):
        tc = dict(lpt.work_items(lens, anchors, bs, C, heads[0], heads[1], q_slice=q_slice, fwd_tile_cost=True))
        pc = dict(lpt.work_items(lens, anchors, bs, C, heads[0], heads[1], q_slice=q_slice))
        assert {k for k, v in pc.items() if v} == {k for k, v in tc.items() if v}
        for key, cost in pc.items():
            assert tc[key] >= cost, (q_slice, key)


def test_forward_tile_cost_equals_pair_cost_for_full_aligned_tiles():
    # one block per 128-row tile, every interval whole key tiles, tiles of a pair alike
    lens, bs, C = [1024], 16, 256
    anchors = [512, 512, 768, 768]
    for q_slice in (0, 1, 2):
        tc = dict(lpt.work_items(lens, anchors, bs, C, 8, 1, q_slice=q_slice, fwd_tile_cost=True))
        pc = dict(lpt.work_items(lens, anchors, bs, C, 8, 1, q_slice=q_slice))
        assert {k: v for k, v in tc.items() if v} == {k: v for k, v in pc.items() if v}
