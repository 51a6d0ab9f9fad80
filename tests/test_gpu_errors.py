"""Bad arguments come back as status codes from host-side checks; no kernel is given a bad pointer."""

import pytest

from gpu_util import small, to_dev

pytestmark = pytest.mark.gpu


def test_host_checks_before_launch(splitkv):
    import torch
    skv = splitkv
    w = small(Hq=4, Hkv=1, d=64)
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.kv_chunk, 148)
    t = {n: to_dev(b) for n, b in w.bits.items()}
    ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
    with pytest.raises(skv.SplitKVError) as ei:          # no device copy yet
        skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws)
    assert ei.value.status == -6
    plan.upload()
    with pytest.raises(skv.SplitKVError) as ei:          # workspace one byte short
        skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws[:-1])
    assert ei.value.status == -3
    lib = skv._lib
    q = t["q"].data_ptr()
    st = lib.splitkv_attn_fwd(plan.handle, q + 2, t["k"].data_ptr(), t["v"].data_ptr(), 1.0, ws.data_ptr(),
                              ws.numel(), None)
    assert st == -1                                       # misaligned q
    st = lib.splitkv_attn_fwd(plan.handle, None, t["k"].data_ptr(), t["v"].data_ptr(), 1.0, ws.data_ptr(),
                              ws.numel(), None)
    assert st == -1                                       # NULL q
    o = torch.empty((w.num_queries, 4, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        skv.splitkv_merge(plan, t["q"], t["kb"], t["vb"], w.scale, ws, o,
                          torch.empty((w.num_queries, 4), device="cuda"))
    st = lib.splitkv_merge(plan.handle, q, t["kb"].data_ptr(), t["vb"].data_ptr(), 1.0, ws.data_ptr(),
                           ws.numel(), o.data_ptr(), 7, o.data_ptr(), None)
    assert st == -1                                       # unknown o dtype
    # the context still works afterwards
    skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws)
    torch.cuda.synchronize()


def test_unsupported_head_dim(splitkv):
    import torch
    skv = splitkv
    w = small(Hq=2, Hkv=1, d=64)
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, 2, 1, 96, w.kv_chunk, 148)
    plan.upload()
    ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
    q = torch.zeros((w.num_queries, 2, 96), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((w.context_len, 1, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(skv.SplitKVError) as ei:            # right sizes: the library refuses d = 96
        skv.splitkv_attn_fwd(plan, q, kv, kv, 1.0, ws)
    assert ei.value.status == -2
    torch.cuda.synchronize()


def test_a_wait_nothing_completes_times_out_and_the_context_survives(splitkv):
    """Failure detection without a fault: a bounded wait on a barrier no one completes gives
    up after its limit and reports SPLITKV_ERR_TIMEOUT with its site; afterwards the same
    context runs a forward and backward that match the oracle."""
    import time
    from gpu_util import TOL_OUT, assert_close, oracle_bwd, run
    t0 = time.time()
    code, site = splitkv.splitkv_selftest_wait_timeout()
    elapsed = time.time() - t0
    assert code == -5                       # SPLITKV_ERR_TIMEOUT
    assert site // 10000 == 9               # a wait of the self-test
    assert 1.5 < elapsed < 60               # the two-second limit, not a hang
    w = small(Hq=4, Hkv=1, d=128)
    out, _, _ = run(w, bwd=True)
    g = oracle_bwd(w)
    assert_close("dq", out["dq"], g["dq"], TOL_OUT)


@pytest.mark.parametrize("claims", [False, True])
def test_waits_past_the_plan_limit_wind_the_attention_kernels_down(splitkv, claims):
    """Failure detection of the attention kernels themselves: under a plan wait limit of 0 a
    wait gives up at the first poll that finds its barrier incomplete.  The forward kernel and
    the two backward kernels then record SPLITKV_ERR_TIMEOUT with the site of the wait, drain
    their copies and products in flight, free their tensor memory and return (no hang, no
    fault); with the default limit restored, the same plan on the same device matches the
    oracle again."""
    import torch
    from context_block_sparse_b200.torch_api import SplitKVAttention
    from gpu_util import TOL_LSE, TOL_OUT, assert_close, oracle_bwd, oracle_fwd
    skv = splitkv
    w = small(Hq=4, Hkv=1, d=128)                      # the smallest shape of the tcgen05 kernels
    t = {n: to_dev(b) for n, b in w.bits.items()}
    att = SplitKVAttention(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                           w.kv_chunk, q_slice=1 if claims else 0, dynamic_claim=claims)
    o, lse = att.forward(t["q"], t["k"], t["v"], t["kb"], t["vb"], w.scale)
    torch.cuda.synchronize()
    skv.splitkv_plan_status(att.plan)                  # a normal run first: no error

    skv.splitkv_plan_set_wait_limit(att.plan, 0)
    att.forward(t["q"], t["k"], t["v"], t["kb"], t["vb"], w.scale)
    torch.cuda.synchronize()
    with pytest.raises(skv.SplitKVError) as ei:
        skv.splitkv_plan_status(att.plan)
    assert ei.value.status == -5 and ei.value.site // 10000 == 1, (ei.value.status, ei.value.site)
    skv.splitkv_plan_status(att.plan)                  # read and cleared
    att.backward(t["q"], t["k"], t["v"], t["kb"], t["vb"], o, lse, t["dout"], w.scale)
    torch.cuda.synchronize()
    with pytest.raises(skv.SplitKVError) as ei:
        skv.splitkv_plan_status(att.plan)
    assert ei.value.status == -5 and ei.value.site // 10000 == 2, (ei.value.status, ei.value.site)

    skv.splitkv_plan_set_wait_limit(att.plan, 2_000_000_000)
    o, lse = att.forward(t["q"], t["k"], t["v"], t["kb"], t["vb"], w.scale)
    g = att.backward(t["q"], t["k"], t["v"], t["kb"], t["vb"], o, lse, t["dout"], w.scale)
    torch.cuda.synchronize()
    skv.splitkv_plan_status(att.plan)
    O, L = oracle_fwd(w)
    assert_close("O", o.cpu().numpy().astype("float64"), O, TOL_OUT)
    assert_close("LSE", lse.cpu().numpy().astype("float64"), L, TOL_LSE)
    ref = oracle_bwd(w)
    for n in ("dq", "dk", "dv"):
        assert_close(n, g[n].cpu().numpy().astype("float64"), ref[n], TOL_OUT)


def test_wait_limit_argument_checks(splitkv):
    skv = splitkv
    w = small(Hq=4, Hkv=1, d=128, grad=False)
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.kv_chunk, 148)
    assert skv._lib.splitkv_plan_set_wait_limit(plan.handle, -1) == -1
    assert skv._lib.splitkv_plan_set_wait_limit(plan.handle, 61_000_000_000) == -1
    assert skv._lib.splitkv_plan_set_wait_limit(None, 5) == -1
    assert skv._lib.splitkv_plan_set_wait_limit(plan.handle, 5) == 0
