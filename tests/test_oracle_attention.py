"""Pins of the fp64 attention oracle against things other than itself (CPU only).

* a dense brute force: an explicit boolean mask over every (query, key) of the
  whole problem, built token by token from the rule on the news page ("Why
  short queries change the problem"), then a masked softmax;
* the one-block special case, which is plain dense attention over the
  concatenated keys: torch's scaled_dot_product_attention in float64;
* the exactness claim of the method (news page, "Exchange the smaller side";
  digest Abstract): the merge of partials over ANY split of the keys equals
  unsplit attention;
* gradients: torch autograd through the dense brute force, and central finite
  differences of the oracle's own forward;
* planted mistakes in the oracle are caught by these pins.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import mask


def _problem(seed, Hq=2, Hkv=1, d=8, bs=3, lens=(11, 7, 5), A=5):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    N = int(lens.sum())
    anchors = np.sort(rng.choice(N, size=A, replace=False)).astype(np.int32)
    Nq = A * bs
    t = {
        "q": rng.standard_normal((Nq, Hq, d)),
        "k": rng.standard_normal((N, Hkv, d)),
        "v": rng.standard_normal((N, Hkv, d)),
        "kb": rng.standard_normal((Nq, Hkv, d)),
        "vb": rng.standard_normal((Nq, Hkv, d)),
        "dout": rng.standard_normal((Nq, Hq, d)),
    }
    return lens, anchors, bs, t


def _dense_mask(lens, anchors, bs):
    """Boolean [Nq, N + Nq]: columns are the N context keys, then every block key."""
    tok_sample = []
    for s, L in enumerate(lens):
        tok_sample += [s] * int(L)
    N = len(tok_sample)
    Nq = len(anchors) * bs
    M = np.zeros((Nq, N + Nq), dtype=bool)
    for i in range(Nq):
        b = i // bs
        a = int(anchors[b])
        for j in range(N):
            M[i, j] = tok_sample[j] == tok_sample[a] and j < a
        for i2 in range(Nq):
            M[i, N + i2] = (i2 // bs) == b
    return M


def _dense_fwd_torch(q, k, v, kb, vb, M, scale):
    """Masked softmax attention over all keys at once (torch float64)."""
    Nq, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    keys = torch.cat([k, kb], dim=0)            # [N+Nq, Hkv, d]
    vals = torch.cat([v, vb], dim=0)
    Mt = torch.as_tensor(M)
    outs, lses = [], []
    for h in range(Hq):
        s = scale * q[:, h, :] @ keys[:, h // G, :].T
        s = s.masked_fill(~Mt, -math.inf)
        lse = torch.logsumexp(s, dim=1)
        p = torch.exp(s - lse[:, None])
        outs.append(p @ vals[:, h // G, :])
        lses.append(lse)
    return torch.stack(outs, dim=1), torch.stack(lses, dim=1)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("heads", [(1, 1), (2, 1), (4, 2)])
def test_fwd_matches_dense_brute_force(seed, heads):
    Hq, Hkv = heads
    lens, anchors, bs, t = _problem(seed, Hq=Hq, Hkv=Hkv)
    scale = 0.37
    O, LSE = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale)
    M = _dense_mask(lens, anchors, bs)
    Ot, Lt = _dense_fwd_torch(*(torch.tensor(t[n]) for n in ("q", "k", "v", "kb", "vb")), M, scale)
    np.testing.assert_allclose(O, Ot.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, Lt.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("rel", [0, 1, 9, 10])
def test_single_block_is_textbook_attention(rel):
    """One block at offset rel: dense attention of its bs rows over [K[S:S+rel]; Kb]."""
    rng = np.random.default_rng(rel)
    lens = np.asarray([6, 11], dtype=np.int32)
    S = 6
    anchors = np.asarray([S + rel], dtype=np.int32)
    bs, d = 4, 16
    q = rng.standard_normal((bs, 1, d))
    k = rng.standard_normal((17, 1, d))
    v = rng.standard_normal((17, 1, d))
    kb = rng.standard_normal((bs, 1, d))
    vb = rng.standard_normal((bs, 1, d))
    scale = 1.0 / math.sqrt(d)
    O, LSE = att.attention_fwd(q, k, v, kb, vb, lens, anchors, bs, scale)
    keys = torch.tensor(np.concatenate([k[S:S + rel, 0], kb[:, 0]]))
    vals = torch.tensor(np.concatenate([v[S:S + rel, 0], vb[:, 0]]))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q[:, 0])[None, None], keys[None, None], vals[None, None], scale=scale)[0, 0]
    np.testing.assert_allclose(O[:, 0], ref.numpy(), rtol=0, atol=1e-12)
    lse_ref = torch.logsumexp(scale * torch.tensor(q[:, 0]) @ keys.T, dim=1)
    np.testing.assert_allclose(LSE[:, 0], lse_ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(3))
def test_split_invariance_every_chunk_size(seed):
    """Merged chunk partials equal unsplit attention for every chunk length 1..N."""
    lens, anchors, bs, t = _problem(seed, Hq=2, Hkv=1, d=4, lens=(9, 6), A=4)
    N = int(lens.sum())
    args = (t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs)
    O, LSE = att.attention_fwd(*args, 0.5)
    for C in range(1, N + 1):
        Os, Ls = att.split_fwd(*args, C, 0.5)
        np.testing.assert_allclose(Os, O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(Ls, LSE, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(10))
def test_merge_over_random_key_splits(seed):
    """The merge is exact for any partition of one row set's keys, empty parts included."""
    rng = np.random.default_rng(seed)
    rows, n, d = 3, 13, 5
    s = rng.standard_normal((rows, n)) * 3
    vals = rng.standard_normal((n, d))
    m_all, l_all, O_all = att.partial(s, vals)
    parts = rng.integers(0, 5, size=n)      # 5 parts, some possibly empty
    recs = [att.partial(s[:, parts == p], vals[parts == p]) for p in range(5)]
    recs.append(att.partial(s[:, :0], vals[:0]))   # explicitly empty
    O, lse = att.merge(recs)
    np.testing.assert_allclose(O, O_all, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, m_all + np.log(l_all), rtol=0, atol=1e-12)


def test_empty_partial_and_all_empty_row():
    s = np.zeros((2, 0))
    m, l, O = att.partial(s, np.zeros((0, 3)))
    assert np.all(m == -np.inf) and np.all(l == 0) and np.all(O == 0)
    O2, lse2 = att.merge([(m, l, O), (m, l, O)])
    assert np.all(O2 == 0) and np.all(lse2 == -np.inf)
    # an empty record next to a live one changes nothing
    s1 = np.array([[0.3, -1.0]])
    v1 = np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]])
    live = att.partial(s1, v1)
    O3, lse3 = att.merge([(m[:1], l[:1], O[:1]), live])
    np.testing.assert_allclose(O3, live[2], atol=1e-15)
    np.testing.assert_allclose(lse3, live[0] + np.log(live[1]), atol=1e-15)


def test_large_scores_stay_finite():
    s = np.array([[1000.0, 999.0, -1000.0]])
    vals = np.eye(3)
    m, l, O = att.partial(s, vals)
    O2, lse = att.merge([att.partial(s[:, :1], vals[:1]), att.partial(s[:, 1:], vals[1:])])
    assert np.isfinite(O2).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(O2, O, atol=1e-15)


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("heads", [(1, 1), (4, 2)])
def test_bwd_matches_autograd_of_dense_brute_force(seed, heads):
    Hq, Hkv = heads
    lens, anchors, bs, t = _problem(seed, Hq=Hq, Hkv=Hkv)
    scale = 0.29
    g = att.attention_bwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], t["dout"], lens, anchors, bs, scale)
    M = _dense_mask(lens, anchors, bs)
    ts = {n: torch.tensor(t[n], requires_grad=True) for n in ("q", "k", "v", "kb", "vb")}
    O, _ = _dense_fwd_torch(ts["q"], ts["k"], ts["v"], ts["kb"], ts["vb"], M, scale)
    (O * torch.tensor(t["dout"])).sum().backward()
    for n in ("q", "k", "v", "kb", "vb"):
        np.testing.assert_allclose(g["d" + n], ts[n].grad.numpy(), rtol=0, atol=1e-11, err_msg=n)


def test_bwd_matches_finite_differences():
    lens, anchors, bs, t = _problem(7, Hq=2, Hkv=1, d=4, lens=(8, 5), A=3)
    scale = 0.6
    names = ("q", "k", "v", "kb", "vb")
    g = att.attention_bwd(*(t[n] for n in names), t["dout"], lens, anchors, bs, scale)

    def f(tt):
        O, _ = att.attention_fwd(*(tt[n] for n in names), lens, anchors, bs, scale)
        return float((O * t["dout"]).sum())

    rng = np.random.default_rng(0)
    eps = 1e-6
    for n in names:
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in t[n].shape)
            tp = {m: t[m].copy() for m in names}
            tm = {m: t[m].copy() for m in names}
            tp[n][idx] += eps
            tm[n][idx] -= eps
            fd = (f(tp) - f(tm)) / (2 * eps)
            assert abs(fd - g["d" + n][idx]) <= 1e-7 + 1e-6 * abs(fd), (n, idx, fd, g["d" + n][idx])


# ---------------------------------------------------------------------------
# Planted mistakes (in the oracle, on the CPU): the pins above must catch them.
# ---------------------------------------------------------------------------

def _fwd_matches_dense(lens, anchors, bs, t, scale=0.37):
    O, LSE = att.attention_fwd(t["q"], t["k"], t["v"], t["kb"], t["vb"], lens, anchors, bs, scale)
    M = _dense_mask(lens, anchors, bs)
    Ot, Lt = _dense_fwd_torch(*(torch.tensor(t[n]) for n in ("q", "k", "v", "kb", "vb")), M, scale)
    return np.allclose(O, Ot.numpy(), atol=1e-9) and np.allclose(LSE, Lt.numpy(), atol=1e-9)


def test_planted_inclusive_anchor_is_caught(monkeypatch):
    lens, anchors, bs, t = _problem(1)
    assert _fwd_matches_dense(lens, anchors, bs, t)
    orig = mask.context_interval
    monkeypatch.setattr(att, "context_interval",
                        lambda L, A, *rest: [(S, a + 1) for (S, a) in orig(L, A, *rest)])
    assert not _fwd_matches_dense(lens, anchors, bs, t)


def test_planted_wrong_kv_head_is_caught(monkeypatch):
    lens, anchors, bs, t = _problem(2, Hq=4, Hkv=2)
    assert _fwd_matches_dense(lens, anchors, bs, t)
    orig = att._block_keys
    monkeypatch.setattr(att, "_block_keys",
                        lambda k, v, kb, vb, S, a, b, bs_, g, *rest: orig(k, v, kb, vb, S, a, b, bs_, (g + 1) % 2,
                                                                           *rest))
    assert not _fwd_matches_dense(lens, anchors, bs, t)


def test_planted_swapped_key_value_is_caught(monkeypatch):
    lens, anchors, bs, t = _problem(3)
    orig = att._block_keys
    monkeypatch.setattr(att, "_block_keys",
                        lambda k, v, kb, vb, S, a, b, bs_, g, *rest: orig(k, v, vb, kb, S, a, b, bs_, g, *rest))
    assert not _fwd_matches_dense(lens, anchors, bs, t)


def test_planted_merge_without_rescale_is_caught():
    rng = np.random.default_rng(5)
    s = rng.standard_normal((2, 9)) * 4
    vals = rng.standard_normal((9, 3))
    recs = [att.partial(s[:, :4], vals[:4]), att.partial(s[:, 4:], vals[4:])]
    good, _ = att.merge(recs)
    # dropping the exp(m_x - M) factor (a plausible slip) breaks exactness
    bad = sum(r[1][:, None] * r[2] for r in recs) / sum(r[1] for r in recs)[:, None]
    full = att.partial(s, vals)[2]
    np.testing.assert_allclose(good, full, atol=1e-12)
    assert not np.allclose(bad, full, atol=1e-6)
