"""Rank plans of Split-KV over several ranks (C++, through the C ABI) against the oracle:
bit-exact (CPU only).

Chunk ownership follows the pages' device rule (news page, "Balance actual
attention work": LPT on chunk cost with equal chunk counts); a rank's plan is the
plain plan over the chunks it owns (news page, "Exchange the smaller side": each
device works on its own share of the context).  Everything is integer, so the
ownership, the block ranges, the entries, the pair counts and the schedules must
equal the oracle's exactly.
"""

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import context_parallel as ocp
from oracle import lpt as olpt
from oracle import mask as omask
from synth import make_workload


def _shard(skv, lens, anchors, bs, Hq, Hkv, C, W, R, r, Wb=0, q_slice=0, eq=False, rb=False, tc=False):
    return skv.splitkv_plan_shard(lens, anchors, bs, Hq, Hkv, 64, C, W, R, r, num_bwd_workers=Wb, q_slice=q_slice,
                                  equal_count=eq, block_keys_in_context=rb, tile_cost=tc)


def _check_shards(skv, lens, anchors, bs, Hq, Hkv, C, W, R, Wb=0, q_slice=0, eq=False, rb=False, tc=False):
    owner = ocp.chunk_owners(lens, anchors, bs, C, Hq, R, rb)
    full_entries = omask.chunk_entries(lens, anchors, C, bs, rb)
    full_pairs = [int(x) for x in omask.chunk_pairs(lens, anchors, bs, C, rb)]
    union = []
    for r in range(R):
        plan = _shard(skv, lens, anchors, bs, Hq, Hkv, C, W, R, r, Wb, q_slice, eq, rb, tc)
        assert plan.export(skv.EXPORT_CHUNK_OWNER).tolist() == owner
        b_lo, b_hi = ocp.query_shard(len(anchors), R, r)
        assert plan.export(skv.EXPORT_QUERY_SHARD).tolist() == [r, R, b_lo, b_hi]
        ent = plan.export(skv.EXPORT_ENTRIES).reshape(-1, 4).tolist()
        assert sorted(map(tuple, ent)) == sorted(e for e in full_entries if owner[e[0]] == r)
        keys = [(c, lo, hi, b) for (c, b, lo, hi) in ent]
        assert keys == sorted(keys)
        union += [tuple(e) for e in ent]
        mine = [p if owner[c] == r else 0 for c, p in enumerate(full_pairs)]
        assert plan.export(skv.EXPORT_CHUNK_PAIRS).tolist() == mine
        # schedules: LPT over the work items of the owned chunks
        for what, loads_what, workers, qs, mode in (
                (skv.EXPORT_FWD_SCHEDULE, skv.EXPORT_FWD_LOADS, W, q_slice, False),
                (skv.EXPORT_BWD_SCHEDULE, skv.EXPORT_BWD_LOADS, Wb or W, 0, tc)):
            items = [it for it in olpt.work_items(lens, anchors, bs, C, Hq, Hkv, q_slice=qs, block_keys_in_context=rb,
                                                  tile_cost=mode) if owner[it[0][0]] == r]
            lists, loads = olpt.lpt(items, workers, equal_count=eq)
            got = [[] for _ in range(workers)]
            for w, c, g, s, _ in plan.export(what).reshape(-1, 5).tolist():
                got[w].append((c, g, s))
            assert got == [list(l) for l in lists]
            assert plan.export(loads_what).tolist() == loads
        st_ = plan.stats()
        assert st_["context_pairs"] == Hq * sum(mine)
        assert st_["block_pairs"] == (0 if rb else Hq * (b_hi - b_lo) * bs * bs)
        plan.destroy()
    assert sorted(union) == sorted(full_entries)          # every entry on exactly one rank


@settings(max_examples=80, deadline=None)
@given(
    lens=st.lists(st.integers(1, 300), min_size=1, max_size=5),
    n_anchor=st.integers(1, 30),
    heads=st.sampled_from([(1, 1), (2, 1), (4, 2), (8, 2)]),
    bs=st.sampled_from([1, 2, 4, 16]),
    C=st.integers(1, 150),
    W=st.integers(1, 12),
    R=st.integers(1, 6),
    q_slice=st.integers(0, 2),
    eq=st.booleans(),
    rb=st.booleans(),
    tc=st.booleans(),
    seed=st.integers(0, 2 ** 31 - 1),
)
def test_random_shards_bit_exact(splitkv, lens, n_anchor, heads, bs, C, W, R, q_slice, eq, rb, tc, seed):
    Hq, Hkv = heads
    if 128 % ((Hq // Hkv) * bs):
        return
    rng = np.random.default_rng(seed)
    anchors = rng.integers(0, sum(lens), size=n_anchor).tolist()
    _check_shards(splitkv, lens, anchors, bs, Hq, Hkv, C, W, R, q_slice=q_slice, eq=eq, rb=rb, tc=tc and not q_slice)


@pytest.mark.parametrize("R", [2, 4, 8])
def test_bwd_workload_shards_bit_exact(splitkv, R):
    """64k context, 512 blocks of 16, 32 / 8 heads, chunks of 512."""
    w = make_workload("bwd", seed=1004, with_grad=False)
    _check_shards(splitkv, w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.kv_chunk,
                  148, R, tc=True)


def test_one_rank_is_the_plain_plan(splitkv):
    w = make_workload("drafter", seed=1001, with_grad=False)
    args = (w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim, w.kv_chunk, 148)
    a = splitkv.splitkv_plan(*args, q_slice=2)
    b = splitkv.splitkv_plan_shard(*args, 1, 0, q_slice=2)
    for what in range(9):
        assert np.array_equal(a.export(what), b.export(what)), what
    assert b.export(splitkv.EXPORT_CHUNK_OWNER).tolist() == [0] * a.stats()["num_chunks"]
    assert b.export(splitkv.EXPORT_QUERY_SHARD).tolist() == [0, 1, 0, len(w.anchors)]
    assert a.export(splitkv.EXPORT_QUERY_SHARD).tolist() == [0, 1, 0, len(w.anchors)]


def test_zero_cost_chunks_are_owned_and_zero_filled_by_their_owner_only(splitkv):
    # one sample of 1000 tokens, chunks of 100, anchors early: chunks 3..9 have no cost
    lens, anchors = [1000], [150, 220, 290]
    owner = ocp.chunk_owners(lens, anchors, 4, 100, 2, 3)
    assert sorted(owner.count(r) for r in range(3)) == [3, 3, 4]
    for r in range(3):
        p = splitkv.splitkv_plan_shard(lens, anchors, 4, 2, 1, 64, 100, 8, 3, r)
        assert p.export(splitkv.EXPORT_CHUNK_OWNER).tolist() == owner
        p.destroy()


@pytest.mark.parametrize("R,r", [(0, 0), (2, 2), (2, -1), (-3, 0)])
def test_bad_rank_rejected(splitkv, R, r):
    with pytest.raises(splitkv.SplitKVError) as ei:
        splitkv.splitkv_plan_shard([100], [50], 4, 2, 1, 64, 32, 8, R, r)
    assert ei.value.status == -1


def test_update_keeps_the_rank(splitkv):
    lens = [400, 300]
    a0, a1 = [10, 399, 500], [200, 650, 690, 420]
    p = splitkv.splitkv_plan_shard(lens, a0, 4, 4, 2, 64, 64, 8, 3, 1)
    splitkv.splitkv_plan_update(p, lens, a1)
    q = splitkv.splitkv_plan_shard(lens, a1, 4, 4, 2, 64, 64, 8, 3, 1)
    for what in (*range(9), splitkv.EXPORT_CHUNK_OWNER, splitkv.EXPORT_QUERY_SHARD):
        assert np.array_equal(p.export(what), q.export(what)), what


def test_rank_workspaces_add_up(splitkv):
    w = make_workload("drafter", seed=1001, with_grad=False)
    args = (w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim, w.kv_chunk, 148)
    full = splitkv.splitkv_plan(*args).stats()["num_entries"]
    parts = [splitkv.splitkv_plan_shard(*args, 4, r).stats()["num_entries"] for r in range(4)]
    assert sum(parts) == full and max(parts) < full


@pytest.mark.parametrize("R", [2, 3, 5])
def test_contiguous_rank_ownership_bit_exact(splitkv, R):
    """SPLITKV_FLAG_CONTIGUOUS_RANKS: chunk c to rank floor(c R / n), the rest of each rank
    plan as with LPT ownership."""
    w = make_workload("drafter", seed=1001, with_grad=False)
    args = (w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, 64, w.kv_chunk, 148)
    n = omask.num_chunks(w.context_len, w.kv_chunk)
    owner = ocp.chunk_owners_contiguous(n, R)
    full_entries = omask.chunk_entries(w.sample_lens, w.anchors, w.kv_chunk, w.block_size)
    union = []
    for r in range(R):
        p = splitkv.splitkv_plan_shard(*args, R, r, contiguous_ranks=True)
        assert p.export(splitkv.EXPORT_CHUNK_OWNER).tolist() == owner
        ent = p.export(splitkv.EXPORT_ENTRIES).reshape(-1, 4).tolist()
        assert sorted(map(tuple, ent)) == sorted(e for e in full_entries if owner[e[0]] == r)
        union += [tuple(e) for e in ent]
        p.destroy()
    assert sorted(union) == sorted(full_entries)
    # a plain plan ignores the flag
    a = splitkv.splitkv_plan(*args)
    b = splitkv.splitkv_plan(*args, contiguous_ranks=True)
    assert np.array_equal(a.export(splitkv.EXPORT_FWD_SCHEDULE), b.export(splitkv.EXPORT_FWD_SCHEDULE))


def _owner_slot(A, R, bs, src, b, t):
    """The merge kernel's destination of row t of block b sent by rank `src` under
    splitkv_merge_to_owners: (owner, row in the owner's [R][rows_owner] receive buffer)."""
    own = ((b + 1) * R - 1) // A
    lo, hi = (own * A) // R, ((own + 1) * A) // R
    assert lo <= b < hi
    return own, src * (hi - lo) * bs + (b - lo) * bs + t


@pytest.mark.parametrize("bs", [1, 4, 16])
def test_owner_scatter_is_the_all_to_all_layout(bs):
    """Every (sender, row) lands once, at the place the all-to-all of SplitKVContextParallel
    puts it: rank r's rows are blocks [floor(r A / R), floor((r + 1) A / R)), received as
    [sender][row - first row]."""
    from context_block_sparse_b200.context_parallel import block_ranges
    for A in range(1, 40):
        for R in range(1, 10):
            ranges = block_ranges(A, R)
            seen = set()
            for src in range(R):
                for b in range(A):
                    for t in range(bs):
                        own, slot = _owner_slot(A, R, bs, src, b, t)
                        lo, hi = ranges[own]
                        assert lo <= b < hi
                        assert slot == src * (hi - lo) * bs + (b * bs + t - lo * bs)
                        assert 0 <= slot < R * (hi - lo) * bs
                        seen.add((own, slot))
            assert len(seen) == R * A * bs
