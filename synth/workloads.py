"""Synthetic workloads shaped like the Split-KV drafter-training regime.

Source: "Split-KV: Efficient Context Parallelism for Training Diffusion
Drafters" (paper digest page, Abstract; news page, sections "Why short queries
change the problem" and "What the speedups cover").  The pages time on
randomly generated fixed-length samples with a query budget far shorter than
the packed context; they give no distribution for anchors or activations, so
the recipe below is this library's own reading:

* samples: lengths drawn uniformly from [lo, hi] until they reach the context
  length N; the last sample is truncated so the lengths sum to exactly N;
* anchors ("uniform within samples"): drawn without replacement, uniformly over
  every eligible packed position, a position being eligible when its offset
  inside its sample is at least 1 (so each sample receives anchors in
  proportion to its length); sorted ascending; block b is opened by anchors[b];
* anchors ("skewed"): a sample is chosen with probability proportional to
  L_s - 1, the offset is 1 + floor(x * (L_s - 1)) with x ~ Beta(0.5, 2);
  duplicates are redrawn;
* tensors: standard normal float32 draws (optionally multiplied by a constant),
  rounded once to bfloat16 with round-to-nearest-even; both sides consume the
  same bits.

Everything is seeded with numpy's default_rng(seed), seed = 1000 + the
workload's index in CONFIGS.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np


# --------------------------------------------------------------------------
# bfloat16 helpers (pure bit manipulation, no attention arithmetic)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    bias = ((bits >> 16) & 1) + 0x7FFF
    return ((bits + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# Workload definitions
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    index: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    context_len: int
    len_range: Optional[tuple]          # (lo, hi) for random packing
    fixed_lens: Optional[tuple]         # explicit sample lengths
    num_anchors: int
    anchors_per_sample: Optional[int]   # tiny: fixed count per sample
    anchor_dist: str                    # "uniform" | "beta"
    block_size: int
    kv_chunk: int
    value_scale: float                  # multiplies the N(0,1) draws
    backward: bool
    description: str


CONFIGS: Dict[str, Config] = {
    c.name: c
    for c in [
        Config("tiny", 0, 1, 1, 64, 768, None, (512, 256), 8, 4, "uniform",
               16, 128, 1.0, True,
               "2 packed samples (512+256), 8 anchors x 16, 1 head, d=64, chunk 128"),
        Config("drafter", 1, 32, 8, 128, 16384, (1024, 8192), None, 128, None, "uniform",
               16, 256, 1.0 / math.sqrt(128.0), False,
               "drafter layer fwd: 32/8 heads, d=128, N(0,1)/sqrt(128), 16k context, 2048 queries, chunk 256"),
        Config("budget", 2, 32, 8, 128, 65536, (2048, 16384), None, 512, None, "uniform",
               16, 512, 1.0, False,
               "query-budget fwd: 32/8 heads, d=128, 64k context, 8192 queries (sweep 2k/4k/8k), chunk 512"),
        Config("skew", 3, 32, 8, 128, 131072, (4096, 32768), None, 512, None, "beta",
               16, 512, 1.0, False,
               "skewed-cost fwd: 32/8 heads, d=128, 128k context, 8192 queries, Beta(0.5,2) anchors, chunk 512"),
        Config("bwd", 4, 32, 8, 128, 65536, (2048, 16384), None, 512, None, "uniform",
               16, 512, 1.0, True,
               "fwd+bwd: 32/8 heads, d=128, 64k context, 8192 queries, chunk 512, dO ~ N(0,1)"),
    ]
}


def draw_lengths(rng: np.random.Generator, total: int, lo: int, hi: int) -> np.ndarray:
    """Sample lengths uniform in [lo, hi] until they cover `total`; truncate the last."""
    lens = []
    acc = 0
    while acc < total:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, total - acc)
        lens.append(L)
        acc += L
    return np.asarray(lens, dtype=np.int32)


def _starts(lens: np.ndarray) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)


def draw_anchors_uniform(rng: np.random.Generator, lens: np.ndarray, count: int) -> np.ndarray:
    """`count` distinct packed positions, uniform over offsets >= 1 of every sample."""
    starts = _starts(lens)
    eligible = np.concatenate(
        [np.arange(s + 1, s + L, dtype=np.int64) for s, L in zip(starts, lens) if L > 1]
    )
    if count > eligible.size:
        raise ValueError("more anchors than eligible positions")
    pick = rng.choice(eligible.size, size=count, replace=False)
    return np.sort(eligible[pick]).astype(np.int32)


def draw_anchors_per_sample(rng: np.random.Generator, lens: np.ndarray, per_sample: int) -> np.ndarray:
    """`per_sample` distinct offsets >= 1 inside every sample (tiny workload)."""
    starts = _starts(lens)
    out = []
    for s, L in zip(starts, lens):
        offs = rng.choice(np.arange(1, L), size=per_sample, replace=False)
        out.extend((s + offs).tolist())
    return np.sort(np.asarray(out, dtype=np.int64)).astype(np.int32)


def draw_anchors_beta(rng: np.random.Generator, lens: np.ndarray, count: int,
                      a: float = 0.5, b: float = 2.0) -> np.ndarray:
    """Skewed anchors: sample chosen with prob. proportional to L_s - 1, offset
    1 + floor(x (L_s - 1)) with x ~ Beta(a, b); duplicates redrawn."""
    starts = _starts(lens)
    w = np.maximum(lens.astype(np.float64) - 1.0, 0.0)
    w = w / w.sum()
    chosen = set()
    while len(chosen) < count:
        s = int(rng.choice(lens.size, p=w))
        x = float(rng.beta(a, b))
        off = 1 + int(math.floor(x * (int(lens[s]) - 1)))
        off = min(off, int(lens[s]) - 1)
        chosen.add(int(starts[s]) + off)
    return np.sort(np.asarray(sorted(chosen), dtype=np.int64)).astype(np.int32)


@dataclasses.dataclass
class Workload:
    """One seeded problem instance.

    Tensors are held twice: `*_bits` (uint16 bfloat16 bits, what the CUDA path
    uploads) and the float32 widening of the same bits (what the oracle
    consumes after a further widening to float64).
    """

    config: Config
    seed: int
    sample_lens: np.ndarray   # int32 [S]
    anchors: np.ndarray       # int32 [A] global packed positions
    block_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_chunk: int
    scale: float
    bits: Dict[str, np.ndarray]

    @property
    def context_len(self) -> int:
        return int(self.sample_lens.sum())

    @property
    def num_queries(self) -> int:
        return int(self.anchors.size) * self.block_size

    def f32(self, name: str) -> np.ndarray:
        return bf16_bits_to_f32(self.bits[name])

    def f64(self, name: str) -> np.ndarray:
        return self.f32(name).astype(np.float64)


def _normal_bits(rng: np.random.Generator, shape, scale: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return f32_to_bf16_bits(x)


def make_workload(name: str, num_anchors: Optional[int] = None, seed: Optional[int] = None,
                  with_grad: Optional[bool] = None, tensors: bool = True,
                  overrides: Optional[dict] = None) -> Workload:
    """Build the seeded workload `name` (see CONFIGS).

    num_anchors overrides the anchor count (the budget sweep uses 128/256/512);
    overrides may replace any Config field (used for small ragged test shapes).
    """
    cfg = CONFIGS[name]
    if overrides:
        cfg = dataclasses.replace(cfg, **overrides)
    seed = 1000 + cfg.index if seed is None else seed
    rng = np.random.default_rng(seed)
    if cfg.fixed_lens is not None:
        lens = np.asarray(cfg.fixed_lens, dtype=np.int32)
    else:
        lens = draw_lengths(rng, cfg.context_len, *cfg.len_range)
    A = cfg.num_anchors if num_anchors is None else int(num_anchors)
    if cfg.anchors_per_sample is not None:
        anchors = draw_anchors_per_sample(rng, lens, cfg.anchors_per_sample)
    elif cfg.anchor_dist == "beta":
        anchors = draw_anchors_beta(rng, lens, A)
    else:
        anchors = draw_anchors_uniform(rng, lens, A)
    bs, Hq, Hkv, d = cfg.block_size, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    N = int(lens.sum())
    Nq = int(anchors.size) * bs
    bits: Dict[str, np.ndarray] = {}
    if tensors:
        s = cfg.value_scale
        bits["q"] = _normal_bits(rng, (Nq, Hq, d), s)
        bits["k"] = _normal_bits(rng, (N, Hkv, d), s)
        bits["v"] = _normal_bits(rng, (N, Hkv, d), s)
        bits["kb"] = _normal_bits(rng, (Nq, Hkv, d), s)
        bits["vb"] = _normal_bits(rng, (Nq, Hkv, d), s)
        grad = cfg.backward if with_grad is None else with_grad
        if grad:
            bits["dout"] = _normal_bits(rng, (Nq, Hq, d), 1.0)
    return Workload(cfg, seed, lens, anchors, bs, Hq, Hkv, d, cfg.kv_chunk,
                    1.0 / math.sqrt(d), bits)
