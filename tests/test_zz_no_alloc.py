"""The allocation-free forward entry point, splitkv_attn_fwd_static_scratch (GPU).

Callers that may not call cudaMalloc per call (a framework whose caching
allocator holds the device memory, latency-critical loops, plug-ins handed raw
pointers) use this entry point: its partial records live in the library's
static device buffer instead of a caller-allocated workspace.  Its output must
match the workspace path (splitkv_attn_fwd + splitkv_merge) within the parity
tolerances, on consecutive calls that reuse the shared buffer.

This file is collected last, and passes alone in a fresh process as well as
after the other tests.
"""

import ctypes

import numpy as np
import pytest

from gpu_util import TOL_LSE, TOL_OUT, assert_close, small, to_dev
from synth import make_workload

pytestmark = pytest.mark.gpu


def _workspace_path(skv, plan, t, scale):
    import torch
    ws = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device="cuda")
    Nq, Hq, d = t["q"].shape
    o = torch.empty((Nq, Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((Nq, Hq), dtype=torch.float32, device="cuda")
    skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], scale, ws)
    skv.splitkv_merge(plan, t["q"], t["kb"], t["vb"], scale, ws, o, lse)
    return o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _static_call(skv, plan, t, scale, o, lse):
    """One call straight through the C ABI with raw device pointers."""
    import torch
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = skv._lib.splitkv_attn_fwd_static_scratch(
        plan.handle, t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), t["kb"].data_ptr(),
        t["vb"].data_ptr(), ctypes.c_float(scale), o.data_ptr(), skv.DTYPE_F32, lse.data_ptr(), stream)
    assert st == 0, skv._lib.splitkv_error_string(st).decode()
    torch.cuda.synchronize()
    return o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _setup(skv, w):
    t = {n: to_dev(b) for n, b in w.bits.items()}
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.kv_chunk, 148)
    plan.upload()
    assert skv.splitkv_workspace_size(plan, skv.WS_FWD) <= skv.STATIC_SCRATCH_BYTES
    return t, plan


def test_static_scratch_matches_workspace_path_on_consecutive_calls(splitkv):
    import torch
    skv = splitkv
    wa = small(Hq=8, Hkv=2, d=128, grad=False)
    wb = small(Hq=4, Hkv=1, d=64, lens=(900, 1500), anchors=30, seed=5, grad=False)
    ta, pa = _setup(skv, wa)
    tb, pb = _setup(skv, wb)
    ref_a = _workspace_path(skv, pa, ta, wa.scale)
    ref_b = _workspace_path(skv, pb, tb, wb.scale)
    oa = torch.empty(ta["q"].shape, dtype=torch.float32, device="cuda")
    la = torch.empty(ta["q"].shape[:2], dtype=torch.float32, device="cuda")
    ob = torch.empty(tb["q"].shape, dtype=torch.float32, device="cuda")
    lb = torch.empty(tb["q"].shape[:2], dtype=torch.float32, device="cuda")
    for _ in range(2):                      # two calls in a row on the same problem
        o, l = _static_call(skv, pa, ta, wa.scale, oa, la)
        assert_close("O", o, ref_a[0], TOL_OUT)
        assert_close("LSE", l, ref_a[1], TOL_LSE)
    o, l = _static_call(skv, pb, tb, wb.scale, ob, lb)   # another problem over the left-over buffer
    assert_close("O", o, ref_b[0], TOL_OUT)
    assert_close("LSE", l, ref_b[1], TOL_LSE)


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
