"""The allocation-free forward entry point, splitkv_attn_fwd_static_scratch (GPU).

Callers that may not call cudaMalloc per call (a framework whose caching
allocator holds the device memory, latency-critical loops, plug-ins handed raw
pointers) use this entry point: its partial records live in the library's
static device buffer instead of a caller-allocated workspace.  Its output must
match the fp64 oracle within the parity tolerances (2e-2 on O, 1e-3 on LSE)
and the workspace path (splitkv_attn_fwd + splitkv_merge) within the same
tolerances, on consecutive calls that reuse the shared buffer, under each plan
option that changes what the entry point launches: run-time claims (the claim
cursor reset), bf16 partial records (another record size and store map) and
reading B of the block keys (kb and vb passed as NULL).

This file is collected last, and passes alone in a fresh process as well as
after the other tests.
"""

import ctypes

import numpy as np
import pytest

from gpu_util import TOL_LSE, TOL_OUT, assert_close, oracle_fwd, small, to_dev
from synth import make_workload

pytestmark = pytest.mark.gpu


def _workspace_path(skv, plan, t, scale, rb):
    import torch
    ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
    Nq, Hq, d = t["q"].shape
    o = torch.empty((Nq, Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((Nq, Hq), dtype=torch.float32, device="cuda")
    kb, vb = (None, None) if rb else (t["kb"], t["vb"])
    skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], scale, ws)
    skv.splitkv_merge(plan, t["q"], kb, vb, scale, ws, o, lse)
    return o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _static_call(skv, plan, t, scale, o, lse, rb):
    """One call straight through the C ABI with raw device pointers (NULL block keys under reading B)."""
    import torch
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    kb = None if rb else ctypes.c_void_p(t["kb"].data_ptr())
    vb = None if rb else ctypes.c_void_p(t["vb"].data_ptr())
    o.fill_(float("nan"))                   # nothing of an earlier call may survive in the outputs
    lse.fill_(float("nan"))
    st = skv._lib.splitkv_attn_fwd_static_scratch(
        plan.handle, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), kb, vb, ctypes.c_float(scale),
        o.data_ptr(), skv.DTYPE_F32, lse.data_ptr(), stream)
    assert st == 0, skv._lib.splitkv_error_string(st).decode()
    torch.cuda.synchronize()
    skv.splitkv_plan_status(plan)          # raises on an error a kernel recorded
    return o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _setup(skv, w, **flags):
    t = {n: to_dev(b) for n, b in w.bits.items()}
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.kv_chunk, 148, **flags)
    plan.upload()
    assert skv.splitkv_workspace_size(plan, skv.WS_FWD) <= skv.STATIC_SCRATCH_BYTES
    return t, plan


OPTIONS = {
    "default": {},
    "run_time_claims": dict(dynamic_claim=True, q_slice=2),
    "bf16_records": dict(partial_bf16=True),
    "block_keys_in_context": dict(block_keys_in_context=True),
}


@pytest.mark.parametrize("opt", list(OPTIONS))
def test_static_scratch_matches_oracle_and_workspace_path_on_consecutive_calls(splitkv, opt):
    import torch
    skv = splitkv
    flags = OPTIONS[opt]
    rb = bool(flags.get("block_keys_in_context"))
    wa = small(Hq=8, Hkv=2, d=128, grad=False)
    wb = small(Hq=4, Hkv=1, d=64, lens=(900, 1500), anchors=30, seed=5, grad=False)   # another head_dim
    ta, pa = _setup(skv, wa, **flags)
    tb, pb = _setup(skv, wb, **flags)
    want_a = oracle_fwd(wa, rb=rb)
    want_b = oracle_fwd(wb, rb=rb)
    ref_a = _workspace_path(skv, pa, ta, wa.scale, rb)
    ref_b = _workspace_path(skv, pb, tb, wb.scale, rb)
    oa = torch.empty(ta["q"].shape, dtype=torch.float32, device="cuda")
    la = torch.empty(ta["q"].shape[:2], dtype=torch.float32, device="cuda")
    ob = torch.empty(tb["q"].shape, dtype=torch.float32, device="cuda")
    lb = torch.empty(tb["q"].shape[:2], dtype=torch.float32, device="cuda")
    for _ in range(2):                      # two calls in a row on the same problem
        o, l = _static_call(skv, pa, ta, wa.scale, oa, la, rb)
        assert_close("O vs oracle", o, want_a[0], TOL_OUT)
        assert_close("LSE vs oracle", l, want_a[1], TOL_LSE)
        assert_close("O vs workspace path", o, ref_a[0], TOL_OUT)
        assert_close("LSE vs workspace path", l, ref_a[1], TOL_LSE)
    o, l = _static_call(skv, pb, tb, wb.scale, ob, lb, rb)   # another problem over the left-over buffer
    assert_close("O vs oracle", o, want_b[0], TOL_OUT)
    assert_close("LSE vs oracle", l, want_b[1], TOL_LSE)
    assert_close("O vs workspace path", o, ref_b[0], TOL_OUT)
    assert_close("LSE vs workspace path", l, ref_b[1], TOL_LSE)


def test_static_scratch_rejects_problems_beyond_its_size(splitkv):
    import torch
    skv = splitkv
    w = make_workload("drafter", tensors=False)
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.kv_chunk, 148)
    plan.upload()
    assert skv.splitkv_workspace_size(plan, skv.WS_FWD) > skv.STATIC_SCRATCH_BYTES
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    p = x.data_ptr()
    st = skv._lib.splitkv_attn_fwd_static_scratch(plan.handle, p, p, p, p, p, ctypes.c_float(1.0), p,
                                                  skv.DTYPE_F32, p, None)
    assert st == -3                          # refused before any launch
    torch.cuda.synchronize()
