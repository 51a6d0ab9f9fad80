"""No kernel writes outside its buffers: guard bytes after the workspaces and every output.

compute-sanitizer is not used here; instead every buffer a call may write -- the forward and
backward workspaces and o, lse, dq, dk, dv, dkb, dvb -- is the head of a larger allocation
whose tail is filled with a fixed byte pattern, and the pattern must survive a forward and
backward pass.  The results are checked against the oracle too, so the buffers were used.
"""

import numpy as np
import pytest

from gpu_util import TOL_LSE, TOL_OUT, assert_close, oracle_bwd, oracle_fwd, small, to_dev

pytestmark = pytest.mark.gpu

GUARD = 64 * 1024     # bytes of pattern after every buffer
PATTERN = 0xA5


def _guarded(nbytes, dtype, shape):
    """A tensor of `shape` and `dtype` at the head of nbytes + GUARD bytes of pattern."""
    import torch
    buf = torch.full((nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    t = buf[:nbytes].view(dtype).view(shape) if shape is not None else buf[:nbytes]
    return t, buf, nbytes


CASES = {
    "tcgen05_static": dict(w=dict(), plan=dict()),
    "tcgen05_claims_bf16": dict(w=dict(), plan=dict(q_slice=2, tile_cost=True, dynamic_claim=True,
                                                      partial_bf16=True)),
    "tcgen05_d64": dict(w=dict(Hq=4, Hkv=2, d=64), plan=dict()),
    "mma_bs1": dict(w=dict(Hq=2, Hkv=1, d=64, bs=1, anchors=200, C=64), plan=dict()),
    "reading_b": dict(w=dict(Hq=8, Hkv=1), plan=dict(block_keys_in_context=True)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_guard_bytes_survive_forward_and_backward(splitkv, case):
    import torch
    skv = splitkv
    w = small(**CASES[case]["w"])
    rb = CASES[case]["plan"].get("block_keys_in_context", False)
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.kv_chunk, 148, **CASES[case]["plan"])
    plan.upload()
    t = {n: to_dev(b) for n, b in w.bits.items()}
    Nq, N, Hq, Hkv, d = w.num_queries, w.context_len, w.num_q_heads, w.num_kv_heads, w.head_dim
    f32 = torch.float32
    guarded = {}

    def make(name, nbytes, dtype, shape):
        x, buf, n = _guarded(nbytes, dtype, shape)
        guarded[name] = (buf, n)
        return x

    ws_f = make("ws_fwd", skv.splitkv_workspace_size(plan, skv.WS_FWD), torch.uint8, None)
    ws_b = make("ws_bwd", skv.splitkv_workspace_size(plan, skv.WS_BWD), torch.uint8, None)
    o = make("o", Nq * Hq * d * 4, f32, (Nq, Hq, d))
    lse = make("lse", Nq * Hq * 4, f32, (Nq, Hq))
    dq = make("dq", Nq * Hq * d * 4, f32, (Nq, Hq, d))
    dk = make("dk", N * Hkv * d * 4, f32, (N, Hkv, d))
    dv = make("dv", N * Hkv * d * 4, f32, (N, Hkv, d))
    dkb = None if rb else make("dkb", Nq * Hkv * d * 4, f32, (Nq, Hkv, d))
    dvb = None if rb else make("dvb", Nq * Hkv * d * 4, f32, (Nq, Hkv, d))
    kb, vb = (None, None) if rb else (t["kb"], t["vb"])

    skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws_f)
    skv.splitkv_merge(plan, t["q"], kb, vb, w.scale, ws_f, o, lse)
    skv.splitkv_attn_bwd(plan, t["q"], t["k"], t["v"], kb, vb, o, lse, t["dout"], dq, dk, dv, dkb, dvb, w.scale,
                         ws_b)
    torch.cuda.synchronize()
    skv.splitkv_plan_status(plan)

    for name, (buf, n) in guarded.items():
        tail = buf[n:]
        bad = int((tail != PATTERN).sum().item())
        assert bad == 0, f"{name}: {bad} guard bytes changed after the {n}-byte buffer"

    O, L = oracle_fwd(w, rb=rb)
    assert_close("O", o.cpu().numpy().astype(np.float64), O, TOL_OUT)
    assert_close("LSE", lse.cpu().numpy().astype(np.float64), L, TOL_LSE)
    g = oracle_bwd(w, rb=rb)
    for n, x in (("dq", dq), ("dk", dk), ("dv", dv), ("dkb", dkb), ("dvb", dvb)):
        if x is not None:
            assert_close(n, x.cpu().numpy().astype(np.float64), g[n], TOL_OUT)
    plan.destroy()
