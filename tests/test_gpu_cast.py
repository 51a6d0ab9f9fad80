"""splitkv_cast_bf16 (float32 -> bfloat16 of finished result arrays) and the torch wrapper's
bf16 gradient option, on the GPU.

The cast is checked bit for bit against torch's own float32 -> bfloat16 conversion (round to
nearest even) on values that stress it: signed zeros, infinities, NaN, subnormals, the
largest finite floats, and values exactly halfway between two bf16 numbers (ties to even),
for lengths that exercise the 8-wide vector path, its tail and the element-wise path
(misaligned pointers).  The bf16 gradients are then compared with the fp64 oracle at the
fixed tolerance: one more bf16 rounding (relative 2^-9) of each finished fp32 gradient.
"""

import numpy as np
import pytest

from gpu_util import TOL_OUT, assert_close, oracle_bwd, small, to_dev

pytestmark = pytest.mark.gpu


def _stress_values(n, seed):
    import torch
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n).astype(np.float32) * np.float32(3.0)
    special = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-40, -1e-40, 3.4e38, -3.4e38, 1.0, -1.0],
                       dtype=np.float32)
    # halfway between neighbouring bf16 values: bf16 bits b, b + 1 -> float32 bits (b << 16) + 0x8000
    b = rng.integers(0x3000, 0x5000, size=64).astype(np.uint32)
    ties = ((b << 16) + 0x8000).view(np.float32)
    k = min(n, special.size + ties.size)
    pool = np.concatenate([special, ties])[:k]
    idx = rng.choice(n, size=k, replace=False)
    x[idx] = pool
    return torch.from_numpy(x)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 4096, 1000003])
@pytest.mark.parametrize("offset", [0, 1])
def test_cast_matches_torch_rounding(splitkv, n, offset):
    import torch
    x = _stress_values(n + offset, seed=n).cuda()
    src = x[offset:]                                   # offset 1: not 16-byte aligned
    out = torch.empty(n + offset, dtype=torch.bfloat16, device="cuda")[offset:]
    splitkv.splitkv_cast_bf16(src, out)
    ref = src.to(torch.bfloat16)
    torch.cuda.synchronize()
    got_b = out.view(torch.int16).cpu().numpy()
    ref_b = ref.view(torch.int16).cpu().numpy()
    nan = np.isnan(src.cpu().numpy())
    assert np.array_equal(got_b[~nan], ref_b[~nan])
    assert np.isnan(out.float().cpu().numpy()[nan]).all()


def test_cast_empty_and_errors(splitkv):
    import torch
    a = torch.empty(0, dtype=torch.float32, device="cuda")
    b = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    splitkv.splitkv_cast_bf16(a, b)
    with pytest.raises(ValueError):
        splitkv.splitkv_cast_bf16(torch.zeros(4, device="cuda"), torch.zeros(4, device="cuda"))


@pytest.mark.parametrize("case", [dict(Hq=8, Hkv=2, d=128), dict(Hq=2, Hkv=2, d=64, bs=8, anchors=40)])
def test_bf16_gradients_match_oracle(splitkv, case):
    import torch
    from context_block_sparse_b200.torch_api import SplitKVAttention
    w = small(**case)
    att = SplitKVAttention(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                           w.kv_chunk, num_workers=148)
    t = {n: to_dev(b) for n, b in w.bits.items()}
    o, lse = att.forward(t["q"], t["k"], t["v"], t["kb"], t["vb"], w.scale, out_dtype=torch.bfloat16)
    g16 = att.backward(t["q"], t["k"], t["v"], t["kb"], t["vb"], o, lse, t["dout"], w.scale,
                       grad_dtype=torch.bfloat16)
    g32 = att.backward(t["q"], t["k"], t["v"], t["kb"], t["vb"], o, lse, t["dout"], w.scale)
    torch.cuda.synchronize()
    ref = oracle_bwd(w)
    for n in ("dq", "dk", "dv", "dkb", "dvb"):
        assert g16[n].dtype == torch.bfloat16
        # the bf16 gradients are the fp32 ones rounded, exactly
        assert torch.equal(g16[n], g32[n].to(torch.bfloat16))
        assert_close(n, g16[n].float().cpu().numpy().astype(np.float64), ref[n], TOL_OUT)
