"""Helpers of the GPU parity tests: upload a seeded workload, run the library, compare with the oracle."""

from __future__ import annotations

import numpy as np

from oracle import attention as oatt
from synth import make_workload

# Tolerances (max-abs), fixed for this method: bf16 inputs, fp32 accumulation.
TOL_OUT = 2e-2     # O, dQ, dK, dV, dKb, dVb
TOL_LSE = 1e-3     # log-sum-exp


def to_dev(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def small(name="tiny", lens=(700, 1100, 333), anchors=24, Hq=8, Hkv=2, d=128, bs=16, C=256, seed=77,
          grad=True):
    """A small ragged workload: several chunks and tiles, a short last chunk."""
    return make_workload(name, seed=seed, with_grad=grad, overrides=dict(
        fixed_lens=tuple(lens), context_len=int(sum(lens)), num_anchors=anchors, anchors_per_sample=None,
        anchor_dist="uniform", num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, block_size=bs, kv_chunk=C,
        value_scale=1.0))


def run(w, bwd=False, o_dtype="f32", W=148, Wb=0, q_slice=0, equal_count=False, repeat=1, rb=False,
        partial_bf16=False, tile_cost=False, dynamic_claim=False, contiguous_schedule=False):
    """Run plan/fwd/merge (and bwd) on cuda:0; returns numpy outputs (+ the attention object).
    rb: reading B of the block keys (kb, vb not passed; no dkb, dvb)."""
    import torch
    from context_block_sparse_b200.torch_api import SplitKVAttention
    att = SplitKVAttention(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                           w.kv_chunk, num_workers=W, num_bwd_workers=Wb, q_slice=q_slice,
                           equal_count=equal_count, block_keys_in_context=rb, partial_bf16=partial_bf16,
                           tile_cost=tile_cost, dynamic_claim=dynamic_claim, contiguous_schedule=contiguous_schedule)
    t = {n: to_dev(b) for n, b in w.bits.items()}
    kb, vb = (None, None) if rb else (t["kb"], t["vb"])
    odt = torch.float32 if o_dtype == "f32" else torch.bfloat16
    out = {}
    for _ in range(repeat):
        o, lse = att.forward(t["q"], t["k"], t["v"], kb, vb, w.scale, out_dtype=odt)
        out["o"] = o.float().cpu().numpy().astype(np.float64)
        out["lse"] = lse.cpu().numpy().astype(np.float64)
        if bwd:
            g = att.backward(t["q"], t["k"], t["v"], kb, vb, o, lse, t["dout"], w.scale)
            for n, x in g.items():
                if x is not None:
                    out[n] = x.cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    import context_block_sparse_b200 as skv
    skv.splitkv_plan_status(att.plan)
    return out, att, t


def oracle_fwd(w, blocks=None, rb=False):
    return oatt.attention_fwd(w.f64("q"), w.f64("k"), w.f64("v"), w.f64("kb"), w.f64("vb"),
                              w.sample_lens, w.anchors, w.block_size, w.scale, blocks=blocks,
                              block_keys_in_context=rb)


def oracle_bwd(w, blocks=None, rb=False):
    return oatt.attention_bwd(w.f64("q"), w.f64("k"), w.f64("v"), w.f64("kb"), w.f64("vb"), w.f64("dout"),
                              w.sample_lens, w.anchors, w.block_size, w.scale, blocks=blocks,
                              block_keys_in_context=rb)


def max_abs(a, b):
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def assert_close(name, got, want, tol):
    err = max_abs(got, want)
    ref = float(np.max(np.abs(want))) if want.size else 0.0
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    assert err <= tol, f"{name}: max-abs error {err:.3e} > {tol:.1e} (max |oracle| {ref:.3e})"
    return err
