"""Split-KV over ranks on the GPU, through the C ABI, against the fp64 oracle.

One GPU stands in for R ranks, one after another (no rank waits on another):
each rank plan (splitkv_plan_shard) runs the attention kernels on keys and
values that hold only its own chunks (zeros elsewhere), the ranks' results are
combined by splitkv_combine_ranks and their dq shares summed by
splitkv_sum_ranks, and the outputs must match the unsplit oracle at the fixed
tolerances (max-abs 2e-2 on O and the gradients, 1e-3 on LSE).  Guard values in
dk, dv, dkb, dvb show that a rank writes only the rows of its own chunks and
blocks.  The combine and the sum are also checked alone against the oracle's
combine and an fp32 sum in rank order, and SplitKVContextParallel runs end to end
on a one-rank NCCL group.
"""

import numpy as np
import pytest

from gpu_util import TOL_LSE, TOL_OUT, assert_close, oracle_bwd, oracle_fwd, small, to_dev
from oracle import context_parallel as ocp

pytestmark = pytest.mark.gpu

GUARD = 7.0

CASES = {
    "tcgen05_R2": dict(w=dict(), R=2, plan=dict()),
    "tcgen05_R3_claims_bf16": dict(w=dict(), R=3, plan=dict(q_slice=2, tile_cost=True, dynamic_claim=True,
                                                            partial_bf16=True)),
    "d64_R4": dict(w=dict(Hq=4, Hkv=2, d=64), R=4, plan=dict()),
    "chunk_not_dividing_R2": dict(w=dict(Hq=4, Hkv=1, d=128, C=100, lens=(257, 3, 1000, 61)), R=2, plan=dict()),
    "reading_b_R2": dict(w=dict(Hq=8, Hkv=1), R=2, plan=dict(block_keys_in_context=True)),
    "contiguous_ranks_R3": dict(w=dict(), R=3, plan=dict(contiguous_ranks=True, q_slice=1)),
}


def _emulate(skv, w, R, plan_kw):
    import torch
    rb = plan_kw.get("block_keys_in_context", False)
    t = {n: to_dev(b) for n, b in w.bits.items()}
    Nq, N, Hq, Hkv, d = w.num_queries, w.context_len, w.num_q_heads, w.num_kv_heads, w.head_dim
    f32 = dict(dtype=torch.float32, device="cuda")
    args = (w.sample_lens, w.anchors, w.block_size, Hq, Hkv, d, w.kv_chunk, 148)
    plans, keep = [], []
    o_parts = torch.empty((R, Nq, Hq, d), **f32)
    lse_parts = torch.empty((R, Nq, Hq), **f32)
    for r in range(R):
        plan = skv.splitkv_plan_shard(*args, R, r, **plan_kw).upload()
        owner = plan.export(skv.EXPORT_CHUNK_OWNER)
        rows = torch.from_numpy(np.repeat(owner == r, w.kv_chunk)[:N]).cuda()
        k = torch.where(rows[:, None, None], t["k"], torch.zeros_like(t["k"]))
        v = torch.where(rows[:, None, None], t["v"], torch.zeros_like(t["v"]))
        b_lo, b_hi = plan.export(skv.EXPORT_QUERY_SHARD).tolist()[2:]
        if rb:
            kb = vb = None
        else:   # the draft keys of other ranks' blocks are not there either
            kb, vb = torch.zeros_like(t["kb"]), torch.zeros_like(t["vb"])
            kb[b_lo * w.block_size:b_hi * w.block_size] = t["kb"][b_lo * w.block_size:b_hi * w.block_size]
            vb[b_lo * w.block_size:b_hi * w.block_size] = t["vb"][b_lo * w.block_size:b_hi * w.block_size]
        ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
        skv.splitkv_attn_fwd(plan, t["q"], k, v, w.scale, ws)
        skv.splitkv_merge(plan, t["q"], kb, vb, w.scale, ws, o_parts[r], lse_parts[r])
        plans.append((plan, rows, k, v, kb, vb, b_lo, b_hi))
        keep.append(ws)
    o = torch.empty((Nq, Hq, d), **f32)
    lse = torch.empty((Nq, Hq), **f32)
    skv.splitkv_combine_ranks(o_parts, lse_parts, o, lse)
    # backward of every rank with the final o, lse
    dq_parts = torch.empty((R, Nq, Hq, d), **f32)
    dk = torch.full((N, Hkv, d), float("nan"), **f32)
    dv = torch.full((N, Hkv, d), float("nan"), **f32)
    dkb = None if rb else torch.full((Nq, Hkv, d), float("nan"), **f32)
    dvb = None if rb else torch.full((Nq, Hkv, d), float("nan"), **f32)
    bs = w.block_size
    for r, (plan, rows, k, v, kb, vb, b_lo, b_hi) in enumerate(plans):
        g = {n: torch.full(shape, GUARD, **f32) for n, shape in (("dk", (N, Hkv, d)), ("dv", (N, Hkv, d)),
                                                                   ("dkb", (Nq, Hkv, d)), ("dvb", (Nq, Hkv, d)))}
        if rb:
            g["dkb"] = g["dvb"] = None
        ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_BWD), dtype=torch.uint8, device="cuda")
        skv.splitkv_attn_bwd(plan, t["q"], k, v, kb, vb, o, lse, t["dout"], dq_parts[r], g["dk"], g["dv"],
                             g["dkb"], g["dvb"], w.scale, ws)
        torch.cuda.synchronize()
        skv.splitkv_plan_status(plan)
        # nothing outside the rank's chunks / blocks was written
        for n in ("dk", "dv"):
            assert bool((g[n][~rows] == GUARD).all()), f"rank {r} wrote {n} rows of other ranks' chunks"
            (dk if n == "dk" else dv)[rows] = g[n][rows]
        if not rb:
            mine = slice(b_lo * bs, b_hi * bs)
            for n, dst in (("dkb", dkb), ("dvb", dvb)):
                outside = torch.ones(Nq, dtype=torch.bool, device="cuda")
                outside[mine] = False
                assert bool((g[n][outside] == GUARD).all()), f"rank {r} wrote {n} rows of other ranks' blocks"
                dst[mine] = g[n][mine]
    dq = torch.empty((Nq, Hq, d), **f32)
    skv.splitkv_sum_ranks(dq_parts, dq)
    torch.cuda.synchronize()
    out = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "dkb": dkb, "dvb": dvb}
    for plan, *_ in plans:
        plan.destroy()
    return {n: None if x is None else x.cpu().numpy().astype(np.float64) for n, x in out.items()}


@pytest.mark.parametrize("case", list(CASES))
def test_rank_plans_reproduce_unsplit_attention(splitkv, case):
    cfg = CASES[case]
    w = small(**cfg["w"])
    rb = cfg["plan"].get("block_keys_in_context", False)
    out = _emulate(splitkv, w, cfg["R"], cfg["plan"])
    O, L = oracle_fwd(w, rb=rb)
    assert_close("O", out["o"], O, TOL_OUT)
    assert_close("LSE", out["lse"], L, TOL_LSE)
    g = oracle_bwd(w, rb=rb)
    for n in ("dq", "dk", "dv", "dkb", "dvb"):
        if g[n] is not None:
            assert_close(n, out[n], g[n], TOL_OUT)


def test_bwd_workload_over_four_ranks_sampled(splitkv):
    """64k context, 8k queries, 32 / 8 heads over 4 emulated ranks (the bench's run-time
    claims and tile cost): O, LSE, dQ, dKb, dVb on sampled blocks; dK, dV on the keys of
    two chunks, the oracle summing over every block that reads them."""
    from oracle import mask as omask
    from synth import make_workload
    w = make_workload("bwd")
    out = _emulate(splitkv, w, 4, dict(q_slice=2, tile_cost=True, dynamic_claim=True))
    rng = np.random.default_rng(0)
    A, bs = w.anchors.size, w.block_size
    blocks = sorted({0, A - 1, A // 4, A // 2, 3 * A // 4} | set(rng.choice(A, size=4, replace=False).tolist()))
    rows = np.concatenate([np.arange(b * bs, (b + 1) * bs) for b in blocks])
    O, L = oracle_fwd(w, blocks)
    assert_close("O", out["o"][rows], O[rows], TOL_OUT)
    assert_close("LSE", out["lse"][rows], L[rows], TOL_LSE)
    g = oracle_bwd(w, blocks)
    for n in ("dq", "dkb", "dvb"):
        assert_close(n, out[n][rows], g[n][rows], TOL_OUT)
    C = w.kv_chunk
    starts = omask.sample_starts(w.sample_lens) + [w.context_len]
    mid = len(w.sample_lens) // 2
    chunks = sorted({(starts[1] - 1) // C, (starts[mid + 1] - 1) // C})
    iv = omask.context_interval(w.sample_lens, w.anchors)
    readers = [b for b, (S, a) in enumerate(iv) if any(S < (c + 1) * C and a > c * C for c in chunks)]
    g2 = oracle_bwd(w, readers)
    keys = np.concatenate([np.arange(c * C, min((c + 1) * C, w.context_len)) for c in chunks])
    for n in ("dk", "dv"):
        assert_close(n, out[n][keys], g2[n][keys], TOL_OUT)
    for n in ("o", "lse", "dq", "dk", "dv", "dkb", "dvb"):
        assert np.isfinite(out[n]).all(), n


@pytest.mark.parametrize("R,case", [(2, "tcgen05"), (3, "tcgen05"), (3, "d64")])
def test_merge_to_owners_is_the_merge_laid_out_by_owner(splitkv, R, case):
    """splitkv_merge_to_owners (the exchange fused into the merge) stores, for every rank,
    exactly the rows its plain merge writes, each block's rows in its owner's receive buffer
    [R][rows_owner] at the sender's slot (bit for bit); the owners' combines match the
    oracle.  One GPU, so every destination is local memory."""
    import torch
    from context_block_sparse_b200.context_parallel import block_ranges
    skv = splitkv
    w = small() if case == "tcgen05" else small(Hq=4, Hkv=2, d=64)
    t = {n: to_dev(b) for n, b in w.bits.items()}
    Nq, Hq, d, bs = w.num_queries, w.num_q_heads, w.head_dim, w.block_size
    f32 = dict(dtype=torch.float32, device="cuda")
    ranges = block_ranges(w.anchors.size, R)
    n_rows = [(hi - lo) * bs for lo, hi in ranges]
    recv_o = [torch.full((R, n, Hq, d), float("nan"), **f32) for n in n_rows]
    recv_l = [torch.full((R, n, Hq), float("nan"), **f32) for n in n_rows]
    dest_o = torch.tensor([x.data_ptr() for x in recv_o], dtype=torch.int64, device="cuda")
    dest_l = torch.tensor([x.data_ptr() for x in recv_l], dtype=torch.int64, device="cuda")
    args = (w.sample_lens, w.anchors, bs, Hq, w.num_kv_heads, d, w.kv_chunk, 148)
    o_loc = torch.empty((R, Nq, Hq, d), **f32)
    l_loc = torch.empty((R, Nq, Hq), **f32)
    for r in range(R):
        plan = skv.splitkv_plan_shard(*args, R, r).upload()
        ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
        skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws)
        skv.splitkv_merge(plan, t["q"], t["kb"], t["vb"], w.scale, ws, o_loc[r], l_loc[r])
        skv.splitkv_merge_to_owners(plan, t["q"], t["kb"], t["vb"], w.scale, ws, dest_o, dest_l)
        torch.cuda.synchronize()
        skv.splitkv_plan_status(plan)
        plan.destroy()
    O, L = oracle_fwd(w)
    for own, (lo, hi) in enumerate(ranges):
        rows = slice(lo * bs, hi * bs)
        assert torch.equal(recv_o[own], o_loc[:, rows]), f"owner {own}: o rows differ from the plain merge"
        assert torch.equal(recv_l[own], l_loc[:, rows]), f"owner {own}: lse rows differ from the plain merge"
        o = torch.empty((hi - lo) * bs, Hq, d, **f32)
        lse = torch.empty((hi - lo) * bs, Hq, **f32)
        skv.splitkv_combine_ranks(recv_o[own], recv_l[own], o, lse)
        assert_close("O", o.cpu().numpy().astype(np.float64), O[rows], TOL_OUT)
        assert_close("LSE", lse.cpu().numpy().astype(np.float64), L[rows], TOL_LSE)


@pytest.mark.parametrize("R,case", [(2, "tcgen05"), (3, "d64")])
def test_bwd_reduce_to_owners_is_the_reduce_laid_out_by_owner(splitkv, R, case):
    """splitkv_bwd_reduce_to_owners (the dq exchange fused into the dQ reduce) stores every
    rank's dq rows exactly as its plain backward writes them, in the owners' receive buffers
    (bit for bit), and leaves dkb, dvb as the plain backward does; the owners' sums match
    the oracle's dq."""
    import torch
    from context_block_sparse_b200.context_parallel import block_ranges
    skv = splitkv
    w = small() if case == "tcgen05" else small(Hq=4, Hkv=2, d=64)
    t = {n: to_dev(b) for n, b in w.bits.items()}
    Nq, N, Hq, Hkv, d, bs = w.num_queries, w.context_len, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    f32 = dict(dtype=torch.float32, device="cuda")
    args = (w.sample_lens, w.anchors, bs, Hq, Hkv, d, w.kv_chunk, 148)
    plans = [skv.splitkv_plan_shard(*args, R, r).upload() for r in range(R)]
    o_parts = torch.empty((R, Nq, Hq, d), **f32)
    l_parts = torch.empty((R, Nq, Hq), **f32)
    for r, plan in enumerate(plans):
        ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
        skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws)
        skv.splitkv_merge(plan, t["q"], t["kb"], t["vb"], w.scale, ws, o_parts[r], l_parts[r])
    o = torch.empty((Nq, Hq, d), **f32)
    lse = torch.empty((Nq, Hq), **f32)
    skv.splitkv_combine_ranks(o_parts, l_parts, o, lse)
    ranges = block_ranges(w.anchors.size, R)
    recv = [torch.full((R, (hi - lo) * bs, Hq, d), float("nan"), **f32) for lo, hi in ranges]
    dest = torch.tensor([x.data_ptr() for x in recv], dtype=torch.int64, device="cuda")
    dq_loc = torch.empty((R, Nq, Hq, d), **f32)
    for r, plan in enumerate(plans):
        ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_BWD), dtype=torch.uint8, device="cuda")
        z = lambda shape: torch.zeros(shape, **f32)   # noqa: E731
        g1 = {n: z(s) for n, s in (("dk", (N, Hkv, d)), ("dv", (N, Hkv, d)), ("dkb", (Nq, Hkv, d)),
                                   ("dvb", (Nq, Hkv, d)))}
        g2 = {n: z(x.shape) for n, x in g1.items()}
        skv.splitkv_attn_bwd(plan, t["q"], t["k"], t["v"], t["kb"], t["vb"], o, lse, t["dout"], dq_loc[r],
                             g1["dk"], g1["dv"], g1["dkb"], g1["dvb"], w.scale, ws)
        skv.splitkv_bwd_delta(plan, o, t["dout"], ws)
        skv.splitkv_bwd_partial(plan, t["q"], t["k"], t["v"], lse, t["dout"], g2["dk"], g2["dv"], w.scale, ws)
        skv.splitkv_bwd_reduce_to_owners(plan, t["q"], t["kb"], t["vb"], lse, t["dout"], g2["dkb"], g2["dvb"],
                                         w.scale, ws, dest)
        torch.cuda.synchronize()
        skv.splitkv_plan_status(plan)
        for n in ("dkb", "dvb"):
            assert torch.equal(g1[n], g2[n]), n
    g = oracle_bwd(w)
    for own, (lo, hi) in enumerate(ranges):
        rows = slice(lo * bs, hi * bs)
        assert torch.equal(recv[own], dq_loc[:, rows]), f"owner {own}: dq rows differ from the plain backward"
        dq = torch.empty(((hi - lo) * bs, Hq, d), **f32)
        skv.splitkv_sum_ranks(recv[own], dq)
        assert_close("dq", dq.cpu().numpy().astype(np.float64), g["dq"][rows], TOL_OUT)
    for plan in plans:
        plan.destroy()


def test_enable_peer_access_on_one_gpu(splitkv):
    """The current device needs nothing; a device that does not exist is refused."""
    import torch
    splitkv.splitkv_enable_peer_access(torch.cuda.current_device())
    assert splitkv._lib.splitkv_enable_peer_access(torch.cuda.device_count() + 7) == -1
    assert splitkv._lib.splitkv_enable_peer_access(-1) == -1


def test_merge_to_owners_refuses_a_rank_mismatch(splitkv):
    import torch
    skv = splitkv
    w = small()
    plan = skv.splitkv_plan_shard(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads,
                                  w.head_dim, w.kv_chunk, 148, 2, 1).upload()
    t = {n: to_dev(b) for n, b in w.bits.items()}
    ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
    ptrs = torch.zeros(2, dtype=torch.int64, device="cuda")
    st = skv._lib.splitkv_merge_to_owners(plan.handle, t["q"].data_ptr(), t["kb"].data_ptr(), t["vb"].data_ptr(),
                                          0.1, ws.data_ptr(), ws.numel(), 2, 0, ptrs.data_ptr(), ptrs.data_ptr(),
                                          None)
    assert st == -1                                       # the plan is rank 1's, not rank 0's
    st = skv._lib.splitkv_merge_to_owners(plan.handle, t["q"].data_ptr(), t["kb"].data_ptr(), t["vb"].data_ptr(),
                                          0.1, ws.data_ptr(), ws.numel(), 3, 1, ptrs.data_ptr(), ptrs.data_ptr(),
                                          None)
    assert st == -1                                       # of 2 ranks, not 3
    torch.cuda.synchronize()


@pytest.mark.parametrize("R,d,o_bf16", [(1, 128, False), (3, 128, False), (5, 64, True), (8, 128, True)])
def test_combine_kernel_against_oracle(splitkv, R, d, o_bf16):
    import torch
    rng = np.random.default_rng(R * 100 + d)
    rows = 3001
    o_parts = rng.standard_normal((R, rows, d)).astype(np.float32)
    lse_parts = (rng.standard_normal((R, rows)) * 30).astype(np.float32)
    lse_parts[rng.random((R, rows)) < 0.3] = -np.inf           # ranks holding no key of a row
    lse_parts[:, :7] = -np.inf                                  # rows no rank holds a key of
    lse_parts[0, 7:9] = [88.0, -88.0]                          # far above / below the other ranks
    O, L = ocp.combine_ranks(o_parts.astype(np.float64), lse_parts.astype(np.float64))
    dev = lambda a: torch.from_numpy(a).cuda()
    o = torch.empty((rows, d), dtype=torch.bfloat16 if o_bf16 else torch.float32, device="cuda")
    lse = torch.empty((rows,), dtype=torch.float32, device="cuda")
    splitkv.splitkv_combine_ranks(dev(o_parts), dev(lse_parts), o, lse)
    got_o = o.float().cpu().numpy().astype(np.float64)
    got_l = lse.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(L))
    fin = np.isfinite(L)
    assert np.all(got_o[~fin] == 0)
    assert np.abs(got_l[fin] - L[fin]).max() <= 1e-4 * max(1.0, np.abs(L[fin]).max())
    assert np.abs(got_o - O).max() <= (1e-2 if o_bf16 else 1e-5) * max(1.0, np.abs(O).max())


def test_sum_kernel_is_the_fp32_sum_in_rank_order(splitkv):
    import torch
    rng = np.random.default_rng(9)
    R, n = 6, 4 * 100003
    parts = (rng.standard_normal((R, n)) * np.exp(rng.standard_normal((R, n)) * 4)).astype(np.float32)
    want = parts[0].copy()
    for r in range(1, R):
        want = (want + parts[r]).astype(np.float32)
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    splitkv.splitkv_sum_ranks(torch.from_numpy(parts).cuda(), out)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_combine_and_sum_reject_bad_arguments(splitkv):
    import torch
    lib = splitkv._lib
    a = torch.zeros((2, 8, 64), dtype=torch.float32, device="cuda")
    l = torch.zeros((2, 8), dtype=torch.float32, device="cuda")
    o = torch.zeros((8, 64), dtype=torch.float32, device="cuda")
    lo = torch.zeros((8,), dtype=torch.float32, device="cuda")
    assert lib.splitkv_combine_ranks(0, 8, 64, a.data_ptr(), l.data_ptr(), o.data_ptr(), 0, lo.data_ptr(), None) == -1
    assert lib.splitkv_combine_ranks(2, 8, 62, a.data_ptr(), l.data_ptr(), o.data_ptr(), 0, lo.data_ptr(), None) == -1
    assert lib.splitkv_combine_ranks(2, 8, 64, a.data_ptr() + 4, l.data_ptr(), o.data_ptr(), 0, lo.data_ptr(),
                                     None) == -1
    assert lib.splitkv_combine_ranks(2, 8, 64, a.data_ptr(), l.data_ptr(), o.data_ptr(), 5, lo.data_ptr(), None) == -1
    assert lib.splitkv_sum_ranks(2, 6, a.data_ptr(), o.data_ptr(), None) == -1
    assert lib.splitkv_sum_ranks(2, 8, a.data_ptr() + 8, o.data_ptr(), None) == -1
    assert lib.splitkv_sum_ranks(2, 0, None, None, None) == 0


@pytest.mark.parametrize("exchange", ["nccl", "p2p"])
def test_context_parallel_class_on_one_nccl_rank(splitkv, exchange):
    """SplitKVContextParallel end to end (broadcasts, all-to-all or the fused merge with its
    stream barriers, kernels) on a one-rank group, two steps."""
    import socket

    import torch
    import torch.distributed as dist
    from context_block_sparse_b200.context_parallel import SplitKVContextParallel
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        w = small()
        t = {n: to_dev(b) for n, b in w.bits.items()}
        cp = SplitKVContextParallel(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.kv_chunk, q_slice=2, tile_cost=True, dynamic_claim=True,
                                    exchange=exchange)
        assert cp.owned_rows() == [(c * w.kv_chunk, min((c + 1) * w.kv_chunk, w.context_len))
                                   for c in range(-(-w.context_len // w.kv_chunk))]
        for _ in range(2):
            o, lse = cp.forward(t["q"], t["k"], t["v"], t["kb"], t["vb"], w.scale)
            g = cp.backward(t["k"], t["v"], o, lse, t["dout"], w.scale)
        torch.cuda.synchronize()
        O, L = oracle_fwd(w)
        assert_close("O", o.cpu().numpy().astype(np.float64), O, TOL_OUT)
        assert_close("LSE", lse.cpu().numpy().astype(np.float64), L, TOL_LSE)
        ref = oracle_bwd(w)
        for n in ("dq", "dk", "dv", "dkb", "dvb"):
            assert_close(n, g[n].cpu().numpy().astype(np.float64), ref[n], TOL_OUT)
    finally:
        dist.destroy_process_group()
