"""Pins of the oracle's reading B of the block keys (CPU only).

News page, "Why short queries change the problem": each block attends to the
preceding context of its own sample and to all tokens inside the block.  Under
reading B the block's own tokens are the context positions after its anchor,
so every row of block b reads the context keys of its own sample that lie
before a_b + bs (clipped to the sample's end), and no separate block keys.

Pins: a dense mask built token by token from that rule (with a masked softmax
in torch), torch autograd through it, the exactness of the split form over
every chunk length, the pair count in closed form and by a triple loop, a
hand-worked clipping case, and a planted mistake (the end not clipped to the
sample) that the dense pin catches.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import lpt as olpt
from oracle import mask


def _problem(seed, Hq=2, Hkv=1, d=8, bs=3, lens=(11, 7, 5), A=5):
    rng = np.random.default_rng(100 + seed)
    lens = np.asarray(lens, dtype=np.int32)
    N = int(lens.sum())
    anchors = np.sort(rng.choice(N, size=A, replace=False)).astype(np.int32)
    Nq = A * bs
    t = {
        "q": rng.standard_normal((Nq, Hq, d)),
        "k": rng.standard_normal((N, Hkv, d)),
        "v": rng.standard_normal((N, Hkv, d)),
        "dout": rng.standard_normal((Nq, Hq, d)),
    }
    return lens, anchors, bs, t


def _dense_mask_b(lens, anchors, bs):
    """Boolean [Nq, N]: row i of block b reads key j iff j is in b's sample and j < a_b + bs."""
    tok_sample = []
    for s, L in enumerate(lens):
        tok_sample += [s] * int(L)
    N = len(tok_sample)
    Nq = len(anchors) * bs
    M = np.zeros((Nq, N), dtype=bool)
    for i in range(Nq):
        a = int(anchors[i // bs])
        for j in range(N):
            M[i, j] = tok_sample[j] == tok_sample[a] and j < a + bs
    return M


def _dense_fwd_torch(q, k, v, M, scale):
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    Mt = torch.as_tensor(M)
    outs, lses = [], []
    for h in range(Hq):
        s = scale * q[:, h, :] @ k[:, h // G, :].T
        s = s.masked_fill(~Mt, -math.inf)
        lse = torch.logsumexp(s, dim=1)
        outs.append(torch.exp(s - lse[:, None]) @ v[:, h // G, :])
        lses.append(lse)
    return torch.stack(outs, dim=1), torch.stack(lses, dim=1)


def _fwd_b(lens, anchors, bs, t, scale=0.41):
    return att.attention_fwd(t["q"], t["k"], t["v"], None, None, lens, anchors, bs, scale,
                             block_keys_in_context=True)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("heads", [(1, 1), (2, 1), (4, 2)])
def test_fwd_matches_dense_brute_force(seed, heads):
    lens, anchors, bs, t = _problem(seed, Hq=heads[0], Hkv=heads[1])
    O, LSE = _fwd_b(lens, anchors, bs, t)
    Ot, Lt = _dense_fwd_torch(*(torch.tensor(t[n]) for n in ("q", "k", "v")), _dense_mask_b(lens, anchors, bs),
                              0.41)
    np.testing.assert_allclose(O, Ot.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, Lt.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_bwd_matches_autograd(seed):
    lens, anchors, bs, t = _problem(seed, Hq=4, Hkv=2)
    g = att.attention_bwd(t["q"], t["k"], t["v"], None, None, t["dout"], lens, anchors, bs, 0.33,
                          block_keys_in_context=True)
    assert g["dkb"] is None and g["dvb"] is None
    ts = {n: torch.tensor(t[n], requires_grad=True) for n in ("q", "k", "v")}
    O, _ = _dense_fwd_torch(ts["q"], ts["k"], ts["v"], _dense_mask_b(lens, anchors, bs), 0.33)
    (O * torch.tensor(t["dout"])).sum().backward()
    for n in ("q", "k", "v"):
        np.testing.assert_allclose(g["d" + n], ts[n].grad.numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("seed", range(3))
def test_split_invariance_every_chunk_size(seed):
    lens, anchors, bs, t = _problem(seed, Hq=2, Hkv=1, d=4, lens=(9, 6), A=4)
    N = int(lens.sum())
    O, LSE = _fwd_b(lens, anchors, bs, t, 0.5)
    for C in range(1, N + 1):
        Os, Ls = att.split_fwd(t["q"], t["k"], t["v"], None, None, lens, anchors, bs, C, 0.5,
                               block_keys_in_context=True)
        np.testing.assert_allclose(Os, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Ls, LSE, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(8))
def test_pair_count_closed_form_and_loops(seed):
    lens, anchors, bs, _ = _problem(seed, bs=1 + seed % 5)
    starts = np.concatenate([[0], np.cumsum(lens)])
    total = 0
    for a in anchors:
        s = int(np.searchsorted(starts, a, side="right")) - 1
        total += bs * (min(int(a) + bs, int(starts[s + 1])) - int(starts[s]))
    for C in (1, 4, 7, 23):
        pc = mask.chunk_pairs(lens, anchors, bs, C, block_keys_in_context=True)
        assert int(pc.sum()) == total
        assert list(pc) == mask.chunk_pairs_loops(lens, anchors, bs, C, block_keys_in_context=True)


def test_hand_worked_clipping():
    # samples [0, 5) and [5, 12); block size 4
    lens, bs = [5, 7], 4
    iv = mask.context_interval(lens, [3, 5, 6, 11], bs, block_keys_in_context=True)
    assert iv == [(0, 5), (5, 9), (5, 10), (5, 12)]
    # reading A for the same anchors ends at the anchor
    assert mask.context_interval(lens, [3, 5, 6, 11]) == [(0, 3), (5, 5), (5, 6), (5, 11)]
    ent = mask.chunk_entries(lens, [3, 11], 4, bs, block_keys_in_context=True)
    assert ent == [(0, 0, 0, 4), (1, 0, 4, 5), (1, 1, 5, 8), (2, 1, 8, 12)]


def test_planted_unclipped_end_is_caught(monkeypatch):
    lens, anchors, bs = np.asarray([6, 9], dtype=np.int32), np.asarray([4, 13], dtype=np.int32), 4
    rng = np.random.default_rng(7)
    t = {"q": rng.standard_normal((8, 1, 4)), "k": rng.standard_normal((15, 1, 4)),
         "v": rng.standard_normal((15, 1, 4))}
    M = _dense_mask_b(lens, anchors, bs)

    def matches():
        O, _ = _fwd_b(lens, anchors, bs, t)
        Ot, _ = _dense_fwd_torch(*(torch.tensor(t[n]) for n in ("q", "k", "v")), M, 0.41)
        return np.allclose(O, Ot.numpy(), atol=1e-12)

    assert matches()
    starts = mask.sample_starts(lens)
    monkeypatch.setattr(att, "context_interval",
                        lambda L, A, b_, flag: [(starts[s], int(a) + b_)
                                                for s, a in zip(mask.anchor_sample(L, A), A)])
    assert not matches()


def test_lpt_costs_follow_the_reading():
    lens, anchors, bs, _ = _problem(3, Hq=4, Hkv=2, bs=4)
    for q_slice in (0, 1):
        items = olpt.work_items(lens, anchors, bs, 5, 4, 2, q_slice=q_slice, rows_per_tile=8,
                                block_keys_in_context=True)
        assert sum(c for _, c in items) == 4 * int(mask.chunk_pairs(lens, anchors, bs, 5,
                                                                    block_keys_in_context=True).sum())
