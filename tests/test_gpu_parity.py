"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded bf16 inputs.

Tolerances: max-abs 2e-2 on O, dQ, dK, dV, dKb, dVb and 1e-3 on LSE (bf16
inputs, fp32 accumulation).  Small workloads are compared element by element;
the full-size workloads on sampled blocks/keys, which the oracle computes one
by one.
"""

import numpy as np
import pytest

from gpu_util import TOL_LSE, TOL_OUT, assert_close, oracle_bwd, oracle_fwd, run, small
from oracle import mask as omask
from synth import make_workload

pytestmark = pytest.mark.gpu


def _check_fwd(w, out, blocks=None):
    O, L = oracle_fwd(w, blocks)
    if blocks is not None:
        rows = np.concatenate([np.arange(b * w.block_size, (b + 1) * w.block_size) for b in blocks])
        O, L = O[rows], L[rows]
        got_o, got_l = out["o"][rows], out["lse"][rows]
    else:
        got_o, got_l = out["o"], out["lse"]
    e1 = assert_close("O", got_o, O, TOL_OUT)
    e2 = assert_close("LSE", got_l, L, TOL_LSE)
    return e1, e2


def _check_bwd(w, out):
    g = oracle_bwd(w)
    for n in ("dq", "dk", "dv", "dkb", "dvb"):
        assert_close(n, out[n], g[n], TOL_OUT)


def test_tiny_fwd_bwd_elementwise(splitkv):
    w = make_workload("tiny")
    out, _, _ = run(w, bwd=True)
    _check_fwd(w, out)
    _check_bwd(w, out)


SMALL_CASES = {
    "gqa4_d128": dict(Hq=8, Hkv=2, d=128),
    "mha_d64": dict(Hq=2, Hkv=2, d=64),
    "gqa8_d64": dict(Hq=8, Hkv=1, d=64),
    "gqa4_bs8": dict(Hq=4, Hkv=1, d=128, bs=8, anchors=40),
    "bs1_mha": dict(Hq=1, Hkv=1, d=64, bs=1, anchors=300, C=64),
    "bs32_g4": dict(Hq=4, Hkv=1, d=64, bs=32, anchors=10),
    "chunk_not_dividing": dict(Hq=4, Hkv=1, d=128, C=100, lens=(257, 3, 1000, 61)),
    "one_sample": dict(Hq=4, Hkv=2, d=64, lens=(3001,), anchors=20, C=512),
    # tcgen05 path with 8 rows per slot (records leave through per-row stores)
    "g1_bs8_d128": dict(Hq=2, Hkv=2, d=128, bs=8, anchors=40),
    # tcgen05 path with a whole 128-row tile per block (G = 8)
    "gqa8_d128": dict(Hq=8, Hkv=1, d=128),
    # in-block term on the tensor cores: 64 block keys (four 16-key steps), 128 rows
    "bs64_g2_d128": dict(Hq=4, Hkv=2, d=128, bs=64, anchors=8),
    # 32 block keys, 32 rows (one pass of the reduce kernel)
    "bs32_g1_d128": dict(Hq=2, Hkv=2, d=128, bs=32, anchors=12),
    # 128 block keys: the tensor-core reduce with eight 16-key steps (d = 64), and at
    # d = 128 the two-role reduce at its largest shared memory (226 KB) beside the tensor-core merge
    "bs128_g1_d64": dict(Hq=2, Hkv=2, d=64, bs=128, anchors=6),
    "bs128_g1_d128": dict(Hq=2, Hkv=2, d=128, bs=128, anchors=6),
}


@pytest.mark.parametrize("case", list(SMALL_CASES))
def test_small_ragged_fwd_bwd_elementwise(splitkv, case):
    w = small(**SMALL_CASES[case])
    out, _, _ = run(w, bwd=True)
    _check_fwd(w, out)
    _check_bwd(w, out)


@pytest.mark.parametrize("opts", [
    dict(W=7), dict(W=1), dict(W=300, Wb=5), dict(q_slice=1), dict(q_slice=2, equal_count=True),
    dict(o_dtype="bf16"), dict(q_slice=2, tile_cost=True), dict(tile_cost=True, Wb=5),
    dict(dynamic_claim=True), dict(dynamic_claim=True, W=7, Wb=3, q_slice=1), dict(dynamic_claim=True, W=300),
    dict(dynamic_claim=True, W=1, Wb=1, q_slice=2, partial_bf16=True),
    dict(contiguous_schedule=True, q_slice=2, W=37), dict(contiguous_schedule=True, tile_cost=True, Wb=5),
])
def test_schedules_and_options_same_result(splitkv, opts):
    w = small()
    out, _, _ = run(w, bwd=True, **opts)
    _check_fwd(w, out)
    _check_bwd(w, out)


def test_anchor_at_sample_start_and_adjacent_anchors(splitkv):
    """Empty context interval (block sees only its own keys) and neighbouring anchors."""
    w = small(lens=(300, 200), anchors=6, Hq=4, Hkv=1, d=64)
    w.anchors[:] = np.array([0, 1, 2, 299, 300, 301], dtype=np.int32)
    out, _, _ = run(w, bwd=True)
    _check_fwd(w, out)
    _check_bwd(w, out)


def _spiky_keys(w, frac=0.02, factor=16.0, seed=5):
    """A copy of w whose keys at a random `frac` of positions are multiplied by
    `factor` (a power of two: the bf16 values stay exact).  Rows meeting such a
    key after their first key tile see their maximum jump far past any fixed
    headroom, in either half of a key tile."""
    import dataclasses
    from synth.workloads import f32_to_bf16_bits
    k = w.f32("k").copy()
    pos = np.random.default_rng(seed).random(k.shape[0]) < frac
    k[pos] *= np.float32(factor)
    bits = dict(w.bits)
    bits["k"] = f32_to_bf16_bits(k)
    return dataclasses.replace(w, bits=bits)


@pytest.mark.parametrize("d", [64, 128])
def test_large_score_jumps(splitkv, d):
    """O and LSE keep the fixed tolerances (O is a convex combination of V).  The
    gradients grow with the 16x keys (max |dQ| ~ 60); dS enters the dQ and dK
    products as a bf16 operand (relative rounding 2^-9 per element) summed over a
    chunk's keys with cancellation, so their bound scales with their magnitude:
    max-abs error <= max(2e-2, 1e-2 * max |oracle|) -- a dropped term or a wrong
    sign gives errors of order max |oracle|."""
    w = _spiky_keys(small(Hq=8, Hkv=2, d=d, C=512))
    out, _, _ = run(w, bwd=True)
    _check_fwd(w, out)
    g = oracle_bwd(w)
    for n in ("dq", "dk", "dv", "dkb", "dvb"):
        assert_close(n, out[n], g[n], max(TOL_OUT, 1e-2 * float(np.abs(g[n]).max())))


@pytest.mark.parametrize("d", [64, 128])
def test_partial_records_match_oracle_split(splitkv, d):
    """The workspace records (m_c, l_c, O_c) equal the oracle's per-chunk partials."""
    import torch
    from oracle import attention as oatt
    w = small(Hq=4, Hkv=2, d=d)
    _, att, _ = run(w)
    E = att.plan.stats()["num_entries"]
    bs, Hq, d = w.block_size, w.num_q_heads, w.head_dim
    ws = att.ws_fwd.cpu().numpy()
    rows = E * bs * Hq

    def arr(off, n):
        return ws[off:off + 4 * n].view(np.float32)

    o_bytes = -(-rows * d * 4 // 256) * 256
    ml_bytes = -(-rows * 4 // 256) * 256
    O = arr(0, rows * d).reshape(E, bs, Hq, d)
    m = arr(o_bytes, rows).reshape(E, bs, Hq)
    l = arr(o_bytes + ml_bytes, rows).reshape(E, bs, Hq)
    ent = att.plan.export(0).reshape(-1, 4)
    parts = {(p["c"], p["b"]): p for p in oatt.chunk_partials(
        w.f64("q"), w.f64("k"), w.f64("v"), w.sample_lens, w.anchors, bs, w.kv_chunk, w.scale)}
    for e, (c, b, lo, hi) in enumerate(ent.tolist()):
        p = parts[(c, b)]
        assert (p["lo"], p["hi"]) == (lo, hi)
        assert_close("O_c", O[e].astype(np.float64), p["O"], TOL_OUT)
        # compare m + log l (the chunk's log-sum-exp) and m itself
        assert_close("lse_c", (m[e] + np.log(l[e])).astype(np.float64), p["m"] + np.log(p["l"]), TOL_LSE)
        assert_close("m_c", m[e].astype(np.float64), p["m"], TOL_LSE)
    torch.cuda.synchronize()


READING_B_CASES = {
    "gqa4_d128": dict(Hq=8, Hkv=2, d=128),
    "mha_d64": dict(Hq=2, Hkv=2, d=64),
    "g1_bs8_d128": dict(Hq=2, Hkv=2, d=128, bs=8, anchors=40),
    "chunk_not_dividing": dict(Hq=4, Hkv=1, d=128, C=100, lens=(257, 3, 1000, 61)),
}


@pytest.mark.parametrize("case", list(READING_B_CASES))
def test_block_keys_in_context_fwd_bwd(splitkv, case):
    """Reading B of the block keys (plan flag): every row reads its sample's context up to
    min(a_b + bs, sample end); kb, vb are not passed and no dkb, dvb come back."""
    w = small(**READING_B_CASES[case])
    # an anchor within bs of its sample's end, so the interval end is clipped
    starts = np.concatenate([[0], np.cumsum(w.sample_lens)])
    w.anchors[0] = int(starts[1]) - 2
    w.anchors[-1] = int(starts[-1]) - 1
    out, _, _ = run(w, bwd=True, rb=True)
    assert "dkb" not in out and "dvb" not in out
    O, L = oracle_fwd(w, rb=True)
    assert_close("O", out["o"], O, TOL_OUT)
    assert_close("LSE", out["lse"], L, TOL_LSE)
    g = oracle_bwd(w, rb=True)
    for n in ("dq", "dk", "dv"):
        assert_close(n, out[n], g[n], TOL_OUT)


BF16_CASES = {
    "gqa4_d128": dict(Hq=8, Hkv=2, d=128),                           # records by bulk tensor stores
    "gqa4_d64": dict(Hq=8, Hkv=2, d=64),                             # head_dim 64 on the tcgen05 kernels
    "mha_bs16_d64": dict(Hq=1, Hkv=1, d=64),                         # the tiny workload's layout
    "g1_bs8_d128": dict(Hq=2, Hkv=2, d=128, bs=8, anchors=40),      # 8-row slots: per-lane stores
    "gqa8_d128": dict(Hq=8, Hkv=1, d=128),
    "chunk_not_dividing": dict(Hq=4, Hkv=1, d=128, C=100, lens=(257, 3, 1000, 61)),
}


@pytest.mark.parametrize("case", list(BF16_CASES))
def test_partial_bf16_fwd_bwd(splitkv, case):
    """bf16 partial records (plan flag): one more bf16 rounding (relative 2^-9) of each
    O_c and dQ-partial element before the fp32 combine, within the same tolerances."""
    w = small(**BF16_CASES[case])
    out, _, _ = run(w, bwd=True, partial_bf16=True)
    _check_fwd(w, out)
    _check_bwd(w, out)


def test_partial_bf16_records(splitkv):
    """The bf16 O_c records (and fp32 m_c, l_c) match the oracle's per-chunk partials."""
    from oracle import attention as oatt
    w = small(Hq=4, Hkv=2, d=128)
    _, att, _ = run(w, partial_bf16=True)
    E = att.plan.stats()["num_entries"]
    bs, Hq, d = w.block_size, w.num_q_heads, w.head_dim
    ws = att.ws_fwd.cpu().numpy()
    rows = E * bs * Hq
    o_bytes = -(-rows * d * 2 // 256) * 256
    ml_bytes = -(-rows * 4 // 256) * 256
    O = (ws[:rows * d * 2].view(np.uint16).astype(np.uint32) << 16).view(np.float32).reshape(E, bs, Hq, d)
    m = ws[o_bytes:o_bytes + rows * 4].view(np.float32).reshape(E, bs, Hq)
    ent = att.plan.export(0).reshape(-1, 4)
    parts = {(p["c"], p["b"]): p for p in oatt.chunk_partials(
        w.f64("q"), w.f64("k"), w.f64("v"), w.sample_lens, w.anchors, bs, w.kv_chunk, w.scale)}
    for e, (c, b, lo, hi) in enumerate(ent.tolist()):
        p = parts[(c, b)]
        assert_close("O_c", O[e].astype(np.float64), p["O"], TOL_OUT)
        assert_close("m_c", m[e].astype(np.float64), p["m"], TOL_LSE)


# rows of a 128-row tile in slots of G * bs: with G * bs not a multiple of 8 (here bs = 1)
# the forward and backward run on the mma.sync kernels, which offer neither option
MMA_ONLY = dict(Hq=2, Hkv=2, d=64, bs=1, anchors=200, C=64)


def test_partial_bf16_needs_the_tcgen05_path(splitkv):
    w = small(**MMA_ONLY)
    with pytest.raises(splitkv.SplitKVError) as ei:
        run(w, partial_bf16=True)
    assert ei.value.status == -2   # SPLITKV_ERR_UNSUPPORTED


def test_dynamic_claim_needs_the_tcgen05_path(splitkv):
    w = small(**MMA_ONLY)
    with pytest.raises(splitkv.SplitKVError) as ei:
        run(w, dynamic_claim=True)
    assert ei.value.status == -2   # SPLITKV_ERR_UNSUPPORTED


@pytest.mark.parametrize("case", list(BF16_CASES))
def test_dynamic_claim_fwd_bwd(splitkv, case):
    """Items claimed at run time: every item is run exactly once by some CTA, so the
    results equal the oracle's (and repeat bit for bit, whichever CTA ran what)."""
    w = small(**BF16_CASES[case])
    out, _, _ = run(w, bwd=True, dynamic_claim=True, q_slice=2, tile_cost=True)
    _check_fwd(w, out)
    _check_bwd(w, out)
    again, _, _ = run(w, bwd=True, dynamic_claim=True, q_slice=2, tile_cost=True)
    static, _, _ = run(w, bwd=True, q_slice=2, tile_cost=True)
    for n in out:
        assert np.array_equal(out[n], again[n]), n
        assert np.array_equal(out[n], static[n]), n


def test_merge_alone_on_oracle_partials(splitkv):
    """splitkv_merge fed with oracle-computed partial records reproduces the oracle output."""
    import torch
    import context_block_sparse_b200 as skv
    from gpu_util import to_dev
    from oracle import attention as oatt
    w = small(Hq=4, Hkv=1, d=128)
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads,
                            w.head_dim, w.kv_chunk, 148)
    plan.upload()
    E = plan.stats()["num_entries"]
    bs, Hq, d = w.block_size, w.num_q_heads, w.head_dim
    rows = E * bs * Hq
    o_bytes = -(-rows * d * 4 // 256) * 256
    ml_bytes = -(-rows * 4 // 256) * 256
    ws = np.zeros(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=np.uint8)
    parts = {(p["c"], p["b"]): p for p in oatt.chunk_partials(
        w.f64("q"), w.f64("k"), w.f64("v"), w.sample_lens, w.anchors, bs, w.kv_chunk, w.scale)}
    O = ws[:rows * d * 4].view(np.float32).reshape(E, bs, Hq, d)
    m = ws[o_bytes:o_bytes + rows * 4].view(np.float32).reshape(E, bs, Hq)
    l = ws[o_bytes + ml_bytes:o_bytes + ml_bytes + rows * 4].view(np.float32).reshape(E, bs, Hq)
    for e, (c, b, lo, hi) in enumerate(plan.export(0).reshape(-1, 4).tolist()):
        p = parts[(c, b)]
        O[e], m[e], l[e] = p["O"], p["m"], p["l"]
    ws_d = torch.from_numpy(ws).cuda()
    o = torch.empty((w.num_queries, Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.num_queries, Hq), dtype=torch.float32, device="cuda")
    skv.splitkv_merge(plan, to_dev(w.bits["q"]), to_dev(w.bits["kb"]), to_dev(w.bits["vb"]), w.scale, ws_d, o, lse)
    Oref, Lref = oracle_fwd(w)
    assert_close("O", o.cpu().numpy().astype(np.float64), Oref, TOL_OUT)
    assert_close("LSE", lse.cpu().numpy().astype(np.float64), Lref, TOL_LSE)


def test_backward_is_deterministic(splitkv):
    w = small()
    a, _, _ = run(w, bwd=True)
    b, _, _ = run(w, bwd=True)
    for n in ("o", "lse", "dq", "dk", "dv", "dkb", "dvb"):
        assert np.array_equal(a[n], b[n]), n


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the bench times
# ---------------------------------------------------------------------------

def _sample_blocks(w, n=10, seed=0):
    rng = np.random.default_rng(seed)
    A = w.anchors.size
    pick = {0, A - 1} | set(rng.choice(A, size=min(n, A), replace=False).tolist())
    return sorted(pick)


def test_drafter_fwd_full(splitkv):
    w = make_workload("drafter")
    out, _, _ = run(w)
    _check_fwd(w, out)


@pytest.mark.parametrize("anchors", [128, 256, 512])
def test_budget_fwd_sampled(splitkv, anchors):
    w = make_workload("budget", num_anchors=anchors)
    out, _, _ = run(w)
    _check_fwd(w, out, _sample_blocks(w))
    assert np.isfinite(out["o"]).all() and np.isfinite(out["lse"]).all()


def test_bwd_config_dynamic_claim_matches_static(splitkv):
    """The fwd+bwd workload in the bench's launch configuration with run-time claims:
    bit-identical to the static schedule (the static run is checked against the oracle
    in test_bwd_config_sampled), and repeated launches reuse the cursors correctly."""
    w = make_workload("bwd")
    dyn, att, _ = run(w, bwd=True, dynamic_claim=True, q_slice=2, tile_cost=True, repeat=2)
    static, _, _ = run(w, bwd=True, q_slice=2, tile_cost=True)
    for n in dyn:
        assert np.array_equal(dyn[n], static[n]), n
    import context_block_sparse_b200 as skv
    for which in (skv.WS_FWD, skv.WS_BWD):
        t = skv.splitkv_read_cta_times(att.plan, which)
        assert (t > 0).all()


def test_budget_fwd_sampled_bf16_partials(splitkv):
    w = make_workload("budget", num_anchors=512)
    out, _, _ = run(w, partial_bf16=True)
    _check_fwd(w, out, _sample_blocks(w))
    assert np.isfinite(out["o"]).all() and np.isfinite(out["lse"]).all()


def test_skew_fwd_sampled(splitkv):
    w = make_workload("skew")
    out, _, _ = run(w)
    _check_fwd(w, out, _sample_blocks(w))
    assert np.isfinite(out["o"]).all()


def test_bwd_config_sampled(splitkv):
    """fwd+bwd at 64k context / 8k queries in the bench's launch configuration (query slices of
    two tiles, backward LPT by tile cost, run-time claims): O, LSE, dQ, dKb, dVb on sampled
    blocks; dK, dV on the keys of three chunks (the bench's parity chunks: two read by few
    blocks, one read by every block of the shortest sample), with the oracle summing over every
    block that reads them."""
    from bench import parity_chunks
    w = make_workload("bwd")
    out, _, _ = run(w, bwd=True, dynamic_claim=True, q_slice=2, tile_cost=True)
    blocks = _sample_blocks(w, n=6)
    _check_fwd(w, out, blocks)
    g = oracle_bwd(w, blocks)
    bs = w.block_size
    rows = np.concatenate([np.arange(b * bs, (b + 1) * bs) for b in blocks])
    for n in ("dq", "dkb", "dvb"):
        assert_close(n, out[n][rows], g[n][rows], TOL_OUT)
    chunks, readers, keys = parity_chunks(w)
    assert len(chunks) == 3 and len(readers) > 0
    g2 = oracle_bwd(w, readers)
    for n in ("dk", "dv"):
        assert_close(n, out[n][keys], g2[n][keys], TOL_OUT)
    for n in ("dq", "dk", "dv", "dkb", "dvb"):
        assert np.isfinite(out[n]).all(), n


def test_bwd_config_static_schedule_sampled(splitkv):
    """The same workload on the library's default schedule (static worker lists, pair cost,
    no slices): sampled rows and the dK, dV of the parity chunks against the oracle."""
    from bench import parity_chunks
    w = make_workload("bwd")
    out, _, _ = run(w, bwd=True)
    blocks = _sample_blocks(w, n=3, seed=11)
    _check_fwd(w, out, blocks)
    chunks, readers, keys = parity_chunks(w)
    g2 = oracle_bwd(w, readers)
    for n in ("dk", "dv"):
        assert_close(n, out[n][keys], g2[n][keys], TOL_OUT)


def test_cta_timers_recorded(splitkv):
    import context_block_sparse_b200 as skv
    w = make_workload("drafter")
    out, att, _ = run(w)
    t = skv.splitkv_read_cta_times(att.plan, skv.WS_FWD)
    assert t.shape == (148,) and (t > 0).all()


def test_cta_timers_of_every_partial_kernel(splitkv):
    """Forward, dK/dV and dQ kernels each stamp their CTAs (W, Wb and W of them)."""
    import context_block_sparse_b200 as skv
    w = small()
    _, att, _ = run(w, bwd=True, W=11, Wb=5)
    for which, n in ((skv.WS_FWD, 11), (skv.WS_BWD, 5), (skv.TIMES_DQ, 11)):
        t = skv.splitkv_read_cta_times(att.plan, which)
        assert t.shape == (n,) and (t > 0).all(), which
