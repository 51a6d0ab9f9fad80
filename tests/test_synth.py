"""The seeded workload generator produces the shapes and structure it promises (CPU only)."""

import numpy as np
import pytest

from synth import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_workload


def test_bf16_round_trip_and_rne():
    x = np.array([1.0, -2.5, 3.1415927, 1e-3, 65504.0], dtype=np.float32)
    y = bf16_bits_to_f32(f32_to_bf16_bits(x))
    assert np.all(np.abs(y - x) <= np.abs(x) * 2.0 ** -8)
    # ties go to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> 1
    assert bf16_bits_to_f32(f32_to_bf16_bits(np.array([1.0 + 2.0 ** -8], np.float32)))[0] == 1.0
    assert bf16_bits_to_f32(f32_to_bf16_bits(np.array([1.0 + 3 * 2.0 ** -8], np.float32)))[0] == 1.0 + 2.0 ** -6


@pytest.mark.parametrize("name", list(CONFIGS))
def test_structure(name):
    w = make_workload(name, tensors=False)
    cfg = CONFIGS[name]
    assert int(w.sample_lens.sum()) == cfg.context_len
    assert w.anchors.size == cfg.num_anchors
    assert np.all(np.diff(w.anchors) > 0)
    starts = np.concatenate([[0], np.cumsum(w.sample_lens)[:-1]])
    s = np.searchsorted(starts, w.anchors, side="right") - 1
    assert np.all(w.anchors - starts[s] >= 1)           # offset >= 1 inside the sample
    if cfg.len_range is not None:
        lo, hi = cfg.len_range
        assert np.all(w.sample_lens[:-1] >= lo) and np.all(w.sample_lens <= hi)


def test_tiny_tensors_and_determinism():
    a = make_workload("tiny")
    b = make_workload("tiny")
    assert a.bits["q"].shape == (128, 1, 64)
    assert a.bits["k"].shape == (768, 1, 64)
    assert a.bits["kb"].shape == (128, 1, 64)
    for n in a.bits:
        assert np.array_equal(a.bits[n], b.bits[n])
    assert (a.anchors < 512).sum() == 4
