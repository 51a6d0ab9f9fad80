"""Pins of the multi-rank Split-KV oracle (CPU only).

* chunk ownership (news page, "Balance actual attention work": LPT by cost over
  devices, equal chunk counts): hand-worked assignments, counts, and the makespan
  against an exhaustive equal-count optimum;
* a rank's result is attention over exactly the keys it holds: a dense boolean
  mask built token by token, restricted to the rank's chunks and blocks, then a
  masked softmax;
* the exactness claim (news page, "Exchange the smaller side"): the combine of
  the ranks' results over ANY partition of the chunks is unsplit attention, and
  the ranks' backward shares sum to the unsplit gradients (the unsplit oracle is
  itself pinned to brute force and autograd);
* planted mistakes in the combine are caught.
"""

import itertools

import numpy as np
import pytest

from oracle import attention as att
from oracle import context_parallel as cp
from oracle import mask


def _problem(seed, Hq=2, Hkv=1, d=8, bs=3, lens=(23, 9, 14), A=6):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    N = int(lens.sum())
    anchors = np.sort(rng.choice(N, size=A, replace=False)).astype(np.int32)
    Nq = A * bs
    t = {n: rng.standard_normal(s) for n, s in (("q", (Nq, Hq, d)), ("k", (N, Hkv, d)), ("v", (N, Hkv, d)),
                                                ("kb", (Nq, Hkv, d)), ("vb", (Nq, Hkv, d)),
                                                ("dout", (Nq, Hq, d)))}
    return lens, anchors, bs, t


def test_chunk_owners_hand_worked():
    # one sample of 40 tokens, chunks of 10, bs 1, anchors 35 and 12: the intervals
    # [0, 35) and [0, 12) give chunk pairs 20, 12, 10, 5
    lens, anchors = [40], [35, 12]
    assert [int(x) for x in mask.chunk_pairs(lens, anchors, 1, 10)] == [20, 12, 10, 5]
    # order c0, c1, c2, c3; c0 -> 0; c1 -> 1; c2 -> 1 (12 < 20); c3 -> 0 (20 < 22)
    assert cp.chunk_owners(lens, anchors, 1, 10, 1, 2) == [0, 1, 1, 0]
    assert cp.chunk_owners(lens, anchors, 1, 10, 4, 2) == [0, 1, 1, 0]     # heads scale every cost
    # a fifth chunk of no cost still needs an owner: 5 = 2 * 2 + 1, and rank 1 (load 22)
    # is lighter than rank 0 (25)
    assert [int(x) for x in mask.chunk_pairs([50], anchors, 1, 10)] == [20, 12, 10, 5, 0]
    assert cp.chunk_owners([50], anchors, 1, 10, 1, 2) == [0, 1, 1, 0, 1]
    # three ranks, 4 = 3 * 1 + 1: c0 -> 0, c1 -> 1, c2 -> 2, and c3 to the lightest rank,
    # 2 (10), which may still take a second chunk
    assert cp.chunk_owners(lens, anchors, 1, 10, 1, 3) == [0, 1, 2, 2]
    # one rank owns everything
    assert cp.chunk_owners(lens, anchors, 1, 10, 1, 1) == [0, 0, 0, 0]


def _opt_equal_count(costs, R):
    n = len(costs)
    q, r = divmod(n, R)
    best = None
    for assign in itertools.product(range(R), repeat=n):
        cnt = [assign.count(w) for w in range(R)]
        if sorted(cnt) != sorted([q + 1] * r + [q] * (R - r)):
            continue
        loads = [0] * R
        for c, w in enumerate(assign):
            loads[w] += costs[c]
        mk = max(loads)
        best = mk if best is None else min(best, mk)
    return best


@pytest.mark.parametrize("seed", range(25))
def test_chunk_owners_counts_and_bound(seed):
    rng = np.random.default_rng(500 + seed)
    lens = [int(x) for x in rng.integers(5, 30, size=int(rng.integers(1, 4)))]
    N = sum(lens)
    C = int(rng.integers(6, 14))
    n = -(-N // C)
    if n > 8:
        lens, N = [8 * C - 3], 8 * C - 3
        n = 8
    anchors = [int(x) for x in rng.integers(0, N, size=int(rng.integers(1, 6)))]
    bs, Hq = int(rng.integers(1, 4)), int(rng.integers(1, 3))
    R = int(rng.integers(2, 4))
    owner = cp.chunk_owners(lens, anchors, bs, C, Hq, R)
    assert len(owner) == n and all(0 <= o < R for o in owner)
    q, r = divmod(n, R)
    assert sorted(owner.count(w) for w in range(R)) == sorted([q + 1] * r + [q] * (R - r))
    costs = [Hq * p for p in mask.chunk_pairs(lens, anchors, bs, C)]
    loads = [sum(costs[c] for c in range(n) if owner[c] == w) for w in range(R)]
    opt = _opt_equal_count(costs, R)
    assert max(loads) <= (4.0 / 3.0 - 1.0 / (3 * R)) * opt + 1e-9


def test_query_shard_covers_every_block_once():
    for A in (1, 5, 16):
        for R in (1, 2, 3, 7):
            got = [b for r in range(R) for b in range(*cp.query_shard(A, R, r))]
            assert got == list(range(A))


def _rank_dense(lens, anchors, bs, t, scale, C, owner, rank, R):
    """Masked softmax over the dense (query, key) mask restricted to the rank's keys."""
    tok_sample = [s for s, L in enumerate(lens) for _ in range(int(L))]
    N = len(tok_sample)
    A = len(anchors)
    Nq = A * bs
    b_lo, b_hi = cp.query_shard(A, R, rank)
    q, k, v, kb, vb = t["q"], t["k"], t["v"], t["kb"], t["vb"]
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    O = np.zeros(q.shape)
    LSE = np.full(q.shape[:2], -np.inf)
    for i in range(Nq):
        b = i // bs
        a = int(anchors[b])
        for h in range(Hq):
            g = h // G
            keys, vals = [], []
            for j in range(N):
                if tok_sample[j] == tok_sample[a] and j < a and owner[j // C] == rank:
                    keys.append(k[j, g]); vals.append(v[j, g])
            for i2 in range(Nq):
                if i2 // bs == b and b_lo <= b < b_hi:
                    keys.append(kb[i2, g]); vals.append(vb[i2, g])
            if not keys:
                continue
            s = scale * (np.array(keys) @ q[i, h])
            w = np.exp(s - s.max())
            O[i, h] = w @ np.array(vals) / w.sum()
            LSE[i, h] = s.max() + np.log(w.sum())
    return O, LSE


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("R", [2, 3])
def test_rank_result_is_attention_over_its_keys(seed, R):
    lens, anchors, bs, t = _problem(seed)
    C, scale = 7, 0.37
    owner = cp.chunk_owners(lens, anchors, bs, C, 2, R)
    for rank in range(R):
        O, L = cp.rank_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, C, scale, owner, rank, R)
        Od, Ld = _rank_dense(lens, anchors, bs, t, scale, C, owner, rank, R)
        np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
        assert np.array_equal(np.isinf(L), np.isinf(Ld))
        fin = np.isfinite(Ld)
        np.testing.assert_allclose(L[fin], Ld[fin], rtol=0, atol=1e-12)


def _random_owner(rng, n, R):
    return [int(x) for x in rng.integers(0, R, size=n)]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("reading_b", [False, True])
def test_combine_over_any_partition_is_unsplit_attention(seed, reading_b):
    lens, anchors, bs, t = _problem(seed, Hq=4, Hkv=2)
    C, scale = 5, 0.29
    rng = np.random.default_rng(seed)
    n = mask.num_chunks(int(np.sum(lens)), C)
    for R in (1, 2, 3, 5):
        for owner in (cp.chunk_owners(lens, anchors, bs, C, 4, R, reading_b), _random_owner(rng, n, R)):
            parts = [cp.rank_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, C, scale, owner, r, R,
                                 block_keys_in_context=reading_b) for r in range(R)]
            O, L = cp.combine_ranks(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
            Ou, Lu = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale,
                                       block_keys_in_context=reading_b)
            np.testing.assert_allclose(O, Ou, rtol=0, atol=1e-12)
            np.testing.assert_allclose(L, Lu, rtol=0, atol=1e-12)


def test_ranks_without_work_contribute_nothing():
    # 2 chunks on 4 ranks: ranks 2 and 3 hold no chunk; with 2 blocks, ranks 0 and 2 hold none
    lens, anchors, bs, t = _problem(1, lens=(9,), A=2)
    C, scale, R = 5, 0.5, 4
    owner = cp.chunk_owners(lens, anchors, bs, C, 2, R)
    assert sorted(set(owner)) == [0, 1]
    parts = [cp.rank_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, C, scale, owner, r, R)
             for r in range(R)]
    assert cp.query_shard(2, R, 2) == (1, 1)
    assert np.all(parts[2][0] == 0) and np.all(np.isneginf(parts[2][1]))
    O, L = cp.combine_ranks(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    Ou, Lu = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale)
    np.testing.assert_allclose(O, Ou, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lu, rtol=0, atol=1e-12)


def test_combine_of_nothing_is_the_empty_row():
    O, L = cp.combine_ranks(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(O == 0) and np.all(np.isneginf(L))


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("reading_b", [False, True])
def test_backward_shares_sum_to_the_unsplit_gradients(seed, reading_b):
    lens, anchors, bs, t = _problem(seed, Hq=4, Hkv=2)
    C, scale, R = 6, 0.31, 3
    owner = cp.chunk_owners(lens, anchors, bs, C, 4, R, reading_b)
    O, L = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale,
                             block_keys_in_context=reading_b)
    g = att.attention_bwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], t["dout"], lens, anchors, bs, scale,
                          block_keys_in_context=reading_b)
    shares = [cp.rank_bwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], t["dout"], O, L, lens, anchors, bs, C, scale,
                          owner, r, R, block_keys_in_context=reading_b) for r in range(R)]
    np.testing.assert_allclose(sum(s["dq"] for s in shares), g["dq"], rtol=0, atol=1e-12)
    N = int(np.sum(lens))
    for r, s in enumerate(shares):
        mine = np.array([owner[j // C] == r for j in range(N)])
        # a rank's context-key gradients are complete on its chunks and zero elsewhere
        np.testing.assert_allclose(s["dk"][mine], g["dk"][mine], rtol=0, atol=1e-12)
        np.testing.assert_allclose(s["dv"][mine], g["dv"][mine], rtol=0, atol=1e-12)
        assert np.all(s["dk"][~mine] == 0) and np.all(s["dv"][~mine] == 0)
        if not reading_b:
            b_lo, b_hi = cp.query_shard(len(anchors), R, r)
            rows = np.zeros(len(anchors) * bs, dtype=bool)
            rows[b_lo * bs:b_hi * bs] = True
            np.testing.assert_allclose(s["dkb"][rows], g["dkb"][rows], rtol=0, atol=1e-12)
            np.testing.assert_allclose(s["dvb"][rows], g["dvb"][rows], rtol=0, atol=1e-12)
            assert np.all(s["dkb"][~rows] == 0) and np.all(s["dvb"][~rows] == 0)


def test_planted_combine_mistakes_are_caught():
    lens, anchors, bs, t = _problem(2)
    C, scale, R = 5, 0.4, 2
    owner = cp.chunk_owners(lens, anchors, bs, C, 2, R)
    parts = [cp.rank_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, C, scale, owner, r, R)
             for r in range(R)]
    Ou, Lu = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale)
    Op, Lp = np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts])
    # a plain mean of the ranks' outputs (weights dropped)
    assert np.abs(Op.mean(axis=0) - Ou).max() > 1e-3
    # weights exp(LSE_r) without the shift are right in exact arithmetic but the sum of
    # LSE_r instead of their log-sum-exp is not
    assert np.abs(Lp.sum(axis=0) - Lu).max() > 1e-3
    # a combine that lets one rank's row win outright (max instead of softmax weights)
    pick = np.take_along_axis(Op, Lp.argmax(axis=0)[None, :, :, None], axis=0)[0]
    assert np.abs(pick - Ou).max() > 1e-3


def test_contiguous_ownership_hand_worked():
    assert cp.chunk_owners_contiguous(4, 2) == [0, 0, 1, 1]
    assert cp.chunk_owners_contiguous(5, 2) == [0, 0, 0, 1, 1]
    assert cp.chunk_owners_contiguous(7, 3) == [0, 0, 0, 1, 1, 2, 2]
    assert cp.chunk_owners_contiguous(2, 4) == [0, 2]
    for n, R in ((13, 4), (100, 8), (8, 8)):
        own = cp.chunk_owners_contiguous(n, R)
        assert own == sorted(own)                              # in order
        q, r = divmod(n, R)
        assert sorted(own.count(w) for w in range(R)) == sorted([q + 1] * r + [q] * (R - r))


def test_lpt_ownership_beats_contiguous_on_a_skewed_context():
    """All anchors late in a first sample of 2000 tokens, none in the second of 6000: the
    first 8 of 32 chunks carry every pair.  Left in order they all land on rank 0, which
    then holds the whole load; LPT spreads them (the pages' point)."""
    lens = [2000, 6000]
    anchors = list(range(1900, 2000, 5))
    C, R = 250, 4
    pairs = [4 * p for p in mask.chunk_pairs(lens, anchors, 4, C)]
    n = len(pairs)
    loads = lambda own: [sum(pairs[c] for c in range(n) if own[c] == w) for w in range(R)]
    lpt_own = cp.chunk_owners(lens, anchors, 4, C, 4, R)
    con_own = cp.chunk_owners_contiguous(n, R)
    assert max(loads(con_own)) == sum(pairs)
    assert max(loads(con_own)) > 3 * max(loads(lpt_own))


def test_planted_backward_mistake_is_caught():
    """A rank backward that normalises with its own LSE_r instead of the final LSE (a
    plausible slip: each rank has its LSE_r at hand) no longer sums to the unsplit dq."""
    lens, anchors, bs, t = _problem(3, Hq=4, Hkv=2)
    C, scale, R = 6, 0.31, 3
    owner = cp.chunk_owners(lens, anchors, bs, C, 4, R)
    O, L = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale)
    g = att.attention_bwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], t["dout"], lens, anchors, bs, scale)
    right = sum(cp.rank_bwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], t["dout"], O, L, lens, anchors, bs, C,
                            scale, owner, r, R)["dq"] for r in range(R))
    np.testing.assert_allclose(right, g["dq"], rtol=0, atol=1e-12)
    wrong = 0
    for r in range(R):
        O_r, L_r = cp.rank_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, C, scale, owner, r, R)
        L_r = np.where(np.isfinite(L_r), L_r, 0.0)
        wrong = wrong + cp.rank_bwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], t["dout"], O, L_r, lens, anchors,
                                    bs, C, scale, owner, r, R)["dq"]
    assert np.abs(wrong - g["dq"]).max() > 1e-3
