"""Host planner (C++, through the C ABI) against the oracle: bit-exact (CPU only).

Mask metadata and LPT schedules are integer computations, so the library's
entries, pair counts, schedules and loads must equal the oracle's exactly
(news page "Balance actual attention work"; digest Abstract).
"""

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import lpt as olpt
from oracle import mask as omask
from synth import make_workload


def _plan(skv, lens, anchors, bs, Hq, Hkv, d, C, W, Wb=0, q_slice=0, eq=False, rb=False, tc=False, ftc=False,
          dyn=False):
    return skv.splitkv_plan(lens, anchors, bs, Hq, Hkv, d, C, W, num_bwd_workers=Wb, q_slice=q_slice,
                            equal_count=eq, block_keys_in_context=rb, tile_cost=tc, fwd_tile_cost=ftc,
                            dynamic_claim=dyn)


def _check_against_oracle(skv, lens, anchors, bs, Hq, Hkv, C, W, Wb=0, q_slice=0, eq=False, d=64, rb=False,
                          tc=False, ftc=False):
    """rb: reading B of the block keys (block keys in the context); tc / ftc: tile cost of the
    backward / forward schedule."""
    plan = _plan(skv, lens, anchors, bs, Hq, Hkv, d, C, W, Wb, q_slice, eq, rb, tc, ftc)
    G = Hq // Hkv
    # entries: same set per chunk, record order sorted by (lo, hi, block) inside each chunk
    ent = plan.export(skv.EXPORT_ENTRIES).reshape(-1, 4)
    want = omask.chunk_entries(lens, anchors, C, bs, rb)
    assert sorted(map(tuple, ent.tolist())) == sorted(want)
    keys = [(c, lo, hi, b) for (c, b, lo, hi) in ent.tolist()]
    assert keys == sorted(keys)
    # pair counts
    pairs = plan.export(skv.EXPORT_CHUNK_PAIRS)
    assert pairs.tolist() == omask.chunk_pairs(lens, anchors, bs, C, rb).tolist()
    # forward schedule (possibly sliced) and backward schedule (whole chunks)
    for what, loads_what, workers, qs, mode, fmode in (
            (skv.EXPORT_FWD_SCHEDULE, skv.EXPORT_FWD_LOADS, W, q_slice, False, ftc),
            (skv.EXPORT_BWD_SCHEDULE, skv.EXPORT_BWD_LOADS, Wb or W, 0, tc, False)):
        items = olpt.work_items(lens, anchors, bs, C, Hq, Hkv, q_slice=qs, rows_per_tile=128,
                                block_keys_in_context=rb, tile_cost=mode, fwd_tile_cost=fmode)
        lists, loads = olpt.lpt(items, workers, equal_count=eq)
        cost = dict(items)
        sched = plan.export(what).reshape(-1, 5)
        got = [[] for _ in range(workers)]
        for w, c, g, s, cst in sched.tolist():
            got[w].append((c, g, s))
            assert cst == cost[(c, g, s)]
        assert got == [list(l) for l in lists]
        assert plan.export(loads_what).tolist() == loads
        # the LPT order itself (the order run-time claims take)
        order_what = skv.EXPORT_FWD_LPT_ORDER if what == skv.EXPORT_FWD_SCHEDULE else skv.EXPORT_BWD_LPT_ORDER
        order = [((c, g, s), cst) for c, g, s, cst in plan.export(order_what).reshape(-1, 4).tolist()]
        assert order == olpt.lpt_order(items)
    # contiguous baseline
    _, cl = olpt.contiguous(olpt.work_items(lens, anchors, bs, C, Hq, Hkv, block_keys_in_context=rb), W)
    assert plan.export(skv.EXPORT_CONTIG_LOADS).tolist() == cl
    st_ = plan.stats()
    assert st_["context_pairs"] == Hq * int(pairs.sum())
    assert st_["block_pairs"] == (0 if rb else Hq * len(anchors) * bs * bs)
    _, fl = olpt.lpt(olpt.work_items(lens, anchors, bs, C, Hq, Hkv, q_slice=q_slice, block_keys_in_context=rb,
                                     fwd_tile_cost=ftc), W, equal_count=eq)
    assert abs(st_["fwd_imbalance"] - olpt.imbalance(fl)) < 1e-12
    assert abs(st_["contig_imbalance"] - olpt.imbalance(cl)) < 1e-12
    plan.destroy()


@settings(max_examples=120, deadline=None)
@given(
    lens=st.lists(st.integers(1, 300), min_size=1, max_size=6),
    n_anchor=st.integers(1, 40),
    heads=st.sampled_from([(1, 1), (2, 1), (4, 1), (4, 2), (8, 2), (32, 8)]),
    bs=st.sampled_from([1, 2, 4, 8, 16]),
    C=st.integers(1, 200),
    W=st.integers(1, 20),
    Wb=st.integers(0, 9),
    q_slice=st.integers(0, 3),
    eq=st.booleans(),
    rb=st.booleans(),
    tc=st.booleans(),
    ftc=st.booleans(),
    seed=st.integers(0, 2 ** 31 - 1),
)
def test_random_problems_bit_exact(splitkv, lens, n_anchor, heads, bs, C, W, Wb, q_slice, eq, rb, tc, ftc, seed):
    Hq, Hkv = heads
    if 128 % ((Hq // Hkv) * bs):
        return
    rng = np.random.default_rng(seed)
    N = sum(lens)
    anchors = rng.integers(0, N, size=n_anchor).astype(np.int32)   # any order, repeats allowed
    _check_against_oracle(splitkv, lens, anchors, bs, Hq, Hkv, C, W, Wb, q_slice, eq, rb=rb, tc=tc, ftc=ftc)


@pytest.mark.parametrize("name", ["tiny", "drafter", "budget", "skew", "bwd"])
@pytest.mark.parametrize("q_slice,eq,rb,tc,ftc", [(0, False, False, False, False), (2, False, False, False, False),
                                                   (0, True, False, False, False), (2, False, True, False, False),
                                                   (2, False, False, True, False), (0, True, False, True, False),
                                                   (2, False, False, True, True), (0, False, True, False, True),
                                                   (1, True, False, False, True)])
def test_workload_plans_bit_exact(splitkv, name, q_slice, eq, rb, tc, ftc):
    w = make_workload(name, tensors=False)
    _check_against_oracle(splitkv, w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads,
                          w.kv_chunk, 148, 0, q_slice, eq, d=w.head_dim, rb=rb, tc=tc, ftc=ftc)


def test_anchor_at_sample_start_and_chunk_straddle(splitkv):
    _check_against_oracle(splitkv, [4, 4, 9], [0, 4, 5, 16, 8], 2, 2, 1, 3, 2)
    # reading B: anchors 3 and 16 sit within bs of their sample's end (clipped)
    _check_against_oracle(splitkv, [4, 4, 9], [0, 3, 5, 16, 8], 2, 2, 1, 3, 2, rb=True)


@pytest.mark.parametrize("bad", [
    dict(lens=[0, 5]), dict(lens=[-1]), dict(anchors=[9]), dict(anchors=[-1]),
    dict(Hq=3, Hkv=2), dict(bs=0), dict(C=0), dict(W=0), dict(Wb=-1), dict(q_slice=-1),
])
def test_invalid_problems_rejected(splitkv, bad):
    a = dict(lens=[5, 4], anchors=[3, 7], bs=4, Hq=2, Hkv=1, d=64, C=4, W=2, Wb=0, q_slice=0)
    a.update(bad)
    with pytest.raises(splitkv.SplitKVError) as ei:
        _plan(splitkv, a["lens"], a["anchors"], a["bs"], a["Hq"], a["Hkv"], a["d"], a["C"], a["W"], a["Wb"],
              a["q_slice"])
    assert ei.value.status == -1


def test_unsupported_tile_shape(splitkv):
    # G * bs must divide the 128-row query tile
    with pytest.raises(splitkv.SplitKVError) as ei:
        _plan(splitkv, [50], [10], 3, 2, 1, 64, 8, 4)
    assert ei.value.status == -2


def test_attention_calls_need_an_uploaded_plan(splitkv):
    """Host-side checks only: a plan without a device copy is refused before any CUDA call."""
    import ctypes
    plan = _plan(splitkv, [64, 64], [10, 70], 16, 1, 1, 64, 32, 4)
    lib = splitkv._lib
    fake = ctypes.c_void_p(16)
    assert lib.splitkv_attn_fwd(plan.handle, fake, fake, fake, 1.0, fake, 1 << 20, None) == -6
    assert lib.splitkv_merge(plan.handle, fake, fake, fake, 1.0, fake, 1 << 20, fake, 0, fake, None) == -6
    assert lib.splitkv_attn_bwd(plan.handle, *([fake] * 6), 0, fake, fake, *([fake] * 5), 1.0, fake, 1 << 20,
                                None) == -6
    assert lib.splitkv_attn_fwd(None, fake, fake, fake, 1.0, fake, 1 << 20, None) == -1
    plan.destroy()


def test_update_in_place_matches_fresh_plan(splitkv):
    w1 = make_workload("drafter", tensors=False)
    w2 = make_workload("drafter", tensors=False, seed=7)
    p = _plan(splitkv, w1.sample_lens, w1.anchors, 16, 32, 8, 128, 256, 148)
    splitkv.splitkv_plan_update(p, w2.sample_lens, w2.anchors)
    q = _plan(splitkv, w2.sample_lens, w2.anchors, 16, 32, 8, 128, 256, 148)
    for what in range(7):
        assert np.array_equal(p.export(what), q.export(what)), what


def test_workspace_sizes(splitkv):
    w = make_workload("tiny", tensors=False)
    p = _plan(splitkv, w.sample_lens, w.anchors, 16, 1, 1, 64, 128, 148)
    E = p.stats()["num_entries"]
    fwd = splitkv.splitkv_workspace_size(p, splitkv.WS_FWD)
    bwd = splitkv.splitkv_workspace_size(p, splitkv.WS_BWD)
    assert fwd >= E * 16 * 1 * 64 * 4 + 2 * E * 16 * 4
    assert bwd >= E * 16 * 64 * 4 + 128 * 4


def test_lpt_beats_contiguous_on_skew(splitkv):
    w = make_workload("skew", tensors=False)
    p = _plan(splitkv, w.sample_lens, w.anchors, 16, 32, 8, 128, 512, 148)
    st_ = p.stats()
    assert st_["fwd_imbalance"] < 0.05
    assert st_["contig_imbalance"] > 1.0


@pytest.mark.parametrize("name", ["bwd", "skew"])
def test_device_regime_report(splitkv, name):
    """The planner in the pages' device regime (news page, "Balance actual attention
    work": imbalance below 1 % with LPT, clearly better than leaving chunks unbalanced)
    on whole (chunk, KV head) items for W = 8 .. 64, as bench.py reports it."""
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("_bench", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    w = make_workload(name, with_grad=False)
    rep = bench.device_lpt_report(splitkv, w)
    assert sorted(rep, key=int) == ["8", "16", "32", "64"]
    for W, row in rep.items():
        assert row["equal_count_imbalance_pct"] < 1.0, (W, row)
        assert row["lpt_imbalance_pct"] < 1.0, (W, row)
        assert row["makespan_ratio"] > 1.1, (W, row)
        assert row["equal_count_plan_us"] > 0 and row["lpt_plan_us"] > 0


def test_dynamic_claim_keeps_the_static_plan(splitkv):
    """SPLITKV_FLAG_DYNAMIC_CLAIM changes how the kernels take the items, not the plan:
    every exported table is the same with and without it."""
    w = make_workload("drafter", tensors=False)
    a = _plan(splitkv, w.sample_lens, w.anchors, 16, 32, 8, 128, 256, 148, q_slice=2)
    b = _plan(splitkv, w.sample_lens, w.anchors, 16, 32, 8, 128, 256, 148, q_slice=2, dyn=True)
    for what in range(9):
        assert np.array_equal(a.export(what), b.export(what)), what
    sa, sb = a.stats(), b.stats()
    sa.pop("plan_us", None)
    sb.pop("plan_us", None)
    assert sa == sb
    a.destroy()
    b.destroy()


def test_unknown_flag_bits_rejected(splitkv):
    """Flags outside SPLITKV_FLAG_* (1, 2, ..., 128) are an invalid argument; each known bit alone
    is accepted; the contiguous schedule (64) refuses the LPT-only bits 1 and 32."""
    import ctypes
    lib = splitkv._lib
    for flags, want in [(1, 0), (2, 0), (4, 0), (8, 0), (16, 0), (32, 0), (63, 0), (64, 0), (64 | 30, 0),
                        (64 | 1, -1), (64 | 32, -1), (128, 0), (255 & ~33, 0), (256, -1), (1 << 31, -1)]:
        p, keep = splitkv._problem([64, 64], [10, 70], 16, 2, 1, 128, 32, 4, 0, 0, False)
        p.flags = flags
        h = ctypes.c_void_p()
        st = lib.splitkv_plan(ctypes.byref(p), ctypes.byref(h))
        assert st == want, (flags, st)
        if st == 0:
            lib.splitkv_plan_destroy(h)


def test_context_at_int32_limit_rejected(splitkv):
    """A packed context of 2^31 tokens or more is refused before anything is allocated."""
    with pytest.raises(splitkv.SplitKVError) as ei:
        _plan(splitkv, [2 ** 30, 2 ** 30], [5, 2 ** 30 + 7], 16, 2, 1, 128, 512, 4)
    assert ei.value.status == -1
    # one token below the limit is a valid problem size (planned here with a small chunk count)
    lens = [2 ** 30, 2 ** 30 - 1]
    plan = _plan(splitkv, lens, [5], 16, 2, 1, 128, 2 ** 28, 4)
    assert plan.stats()["context_pairs"] == 2 * 16 * 5
    plan.destroy()


def test_plan_dump_is_reproducible(splitkv, tmp_path):
    """A dump (problem, stats, every exported table) of two plans of the same problem is
    identical, and its tables are the plan's exports."""
    w = make_workload("drafter", seed=1001, with_grad=False)
    args = (w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim, w.kv_chunk, 148)
    a = splitkv.splitkv_plan(*args, q_slice=2, tile_cost=True, dynamic_claim=True)
    b = splitkv.splitkv_plan(*args, q_slice=2, tile_cost=True, dynamic_claim=True)
    a.dump(str(tmp_path / "a.npz"))
    b.dump(str(tmp_path / "b.npz"))
    da = splitkv.splitkv_plan_load_dump(str(tmp_path / "a.npz"))
    db = splitkv.splitkv_plan_load_dump(str(tmp_path / "b.npz"))
    assert sorted(da) == sorted(db)
    for k in da:
        assert np.array_equal(da[k], db[k]), k
    assert np.array_equal(da["fwd_schedule"], a.export(splitkv.EXPORT_FWD_SCHEDULE))
    assert np.array_equal(da["anchors"], np.asarray(w.anchors, dtype=np.int32))
    assert int(da["problem_flags"]) == splitkv.FLAG_TILE_COST | splitkv.FLAG_DYNAMIC_CLAIM
    assert int(da["stats_num_entries"]) == a.stats()["num_entries"]
    s = splitkv.splitkv_plan_shard(*args, 4, 3)
    s.dump(str(tmp_path / "s.npz"))
    ds = splitkv.splitkv_plan_load_dump(str(tmp_path / "s.npz"))
    assert ds["query_shard"].tolist() == [3, 4, 3 * len(w.anchors) // 4, len(w.anchors)]
    assert np.array_equal(ds["chunk_owner"], s.export(splitkv.EXPORT_CHUNK_OWNER))


def test_costs_above_32_bits_bit_exact(splitkv):
    """Item costs past 2^32 (72 blocks of 16 x 8 heads reading whole chunks of 2^19 keys)
    take the planner's wide sort; the schedules still equal the oracle's."""
    lens = [1 << 21, 1000]
    anchors = [(1 << 21) - 1 - 3 * i for i in range(72)] + [(1 << 21) + 500, 1 << 20]
    C = 1 << 19
    assert max(omask.chunk_pairs(lens, anchors, 16, C)) * 8 > (1 << 32)
    _check_against_oracle(splitkv, lens, anchors, 16, 8, 1, C, 3, q_slice=1)
    _check_against_oracle(splitkv, lens, anchors, 16, 8, 1, C, 2, eq=True)


@pytest.mark.parametrize("seed", range(12))
def test_contiguous_schedule_bit_exact(splitkv, seed):
    """SPLITKV_FLAG_CONTIGUOUS_SCHEDULE: the non-zero-cost items of each schedule in (chunk,
    head, slice) order, item i of n to worker floor(i W / n) -- the oracle's contiguous
    assignment over the same items."""
    rng = np.random.default_rng(300 + seed)
    lens = [int(x) for x in rng.integers(50, 900, size=int(rng.integers(1, 5)))]
    anchors = [int(x) for x in rng.integers(0, sum(lens), size=int(rng.integers(1, 40)))]
    Hq, Hkv = [(4, 1), (8, 2), (2, 2)][seed % 3]
    bs, C = [4, 8, 16][seed % 3], int(rng.integers(16, 300))
    W, Wb, qs = int(rng.integers(1, 40)), int(rng.integers(1, 40)), seed % 3
    tc = bool(seed % 2)
    plan = splitkv.splitkv_plan(lens, anchors, bs, Hq, Hkv, 64, C, W, num_bwd_workers=Wb, q_slice=qs,
                                tile_cost=tc, contiguous_schedule=True)
    for what, loads_what, order_what, workers, q_slice, mode in (
            (splitkv.EXPORT_FWD_SCHEDULE, splitkv.EXPORT_FWD_LOADS, splitkv.EXPORT_FWD_LPT_ORDER, W, qs, False),
            (splitkv.EXPORT_BWD_SCHEDULE, splitkv.EXPORT_BWD_LOADS, splitkv.EXPORT_BWD_LPT_ORDER, Wb, 0, tc)):
        live = [it for it in olpt.work_items(lens, anchors, bs, C, Hq, Hkv, q_slice=q_slice, tile_cost=mode)
                if it[1] > 0]
        lists, loads = olpt.contiguous(live, workers)
        got = [[] for _ in range(workers)]
        for w_, c, g, s, _ in plan.export(what).reshape(-1, 5).tolist():
            got[w_].append((c, g, s))
        assert got == [list(l) for l in lists]
        assert plan.export(loads_what).tolist() == loads
        order = [((c, g, s), cst) for c, g, s, cst in plan.export(order_what).reshape(-1, 4).tolist()]
        assert order == sorted(live)
    plan.destroy()


@pytest.mark.parametrize("other", ["equal_count", "dynamic_claim"])
def test_contiguous_schedule_refuses_lpt_options(splitkv, other):
    with pytest.raises(splitkv.SplitKVError) as ei:
        splitkv.splitkv_plan([500], [100, 300], 4, 2, 1, 64, 64, 8, contiguous_schedule=True, **{other: True})
    assert ei.value.status == -1
