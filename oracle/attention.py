"""Block-sparse anchor attention in float64 (oracle; test infrastructure).

Definitions ([news] "Why short queries change the problem", "Exchange the
smaller side"; [digest] Abstract):

* Layouts: q, dout [Nq, Hq, d]; k, v [N, Hkv, d]; kb, vb [Nq, Hkv, d].  Query
  row i of block b is token i = b*bs + t; query head h reads KV head
  g = h // (Hq // Hkv) (grouped-query attention).
* Allowed keys of every row of block b, head h: the context keys
  j in [S_{s(b)}, a_b) of KV head g, then the bs in-block keys
  kb[b*bs : (b+1)*bs, g] (values likewise).
* Reading B (`block_keys_in_context`): the block's own tokens are the context
  positions after its anchor; the allowed keys are the context keys
  j in [S_{s(b)}, min(a_b + bs, S_{s(b)} + L_{s(b)})) and nothing else (kb, vb
  unused; dkb, dvb returned as None).
* s = scale * q . key; O = softmax(s) . values; LSE = log(sum(exp(s))) (natural
  log).  Gradients are the analytic gradients of O with respect to q, k, v, kb,
  vb contracted with dout.

The split form ([news] "Exchange the smaller side": partial attention against
each key/value shard, combined exactly with normalisation statistics):

* partial of a key subset X: m = max_{j in X} s_j, l = sum exp(s_j - m),
  O_X = sum exp(s_j - m) v_j / l; an empty subset gives (m, l, O) = (-inf, 0, 0);
* merge: M = max m_x, L = sum l_x exp(m_x - M), O = sum l_x exp(m_x - M) O_x / L,
  LSE = M + log L; subsets with l = 0 are skipped, and a row whose subsets are
  all empty gets O = 0, LSE = -inf.
"""

from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np

from .mask import chunk_entries, context_interval

NEG_INF = -np.inf


def _group(Hq: int, Hkv: int) -> int:
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return Hq // Hkv


def _block_keys(k, v, kb, vb, S, a, b, bs, g, in_context=False):
    if in_context:
        return k[S:a, g, :], v[S:a, g, :]
    keys = np.concatenate([k[S:a, g, :], kb[b * bs:(b + 1) * bs, g, :]], axis=0)
    vals = np.concatenate([v[S:a, g, :], vb[b * bs:(b + 1) * bs, g, :]], axis=0)
    return keys, vals


def attention_fwd(q, k, v, kb, vb, sample_lens, anchors, block_size: int, scale: float,
                  blocks: Optional[Iterable[int]] = None, block_keys_in_context: bool = False
                  ) -> Tuple[np.ndarray, np.ndarray]:
    """O [Nq, Hq, d] and LSE [Nq, Hq] by the plain definition (all inputs float64).

    `blocks` restricts the work to some blocks; other rows are left NaN.
    """
    Nq, Hq, d = q.shape
    Hkv = k.shape[1]
    G = _group(Hq, Hkv)
    bs = int(block_size)
    O = np.full((Nq, Hq, d), np.nan)
    LSE = np.full((Nq, Hq), np.nan)
    iv = context_interval(sample_lens, anchors, bs, block_keys_in_context)
    todo = range(len(iv)) if blocks is None else blocks
    for b in todo:
        S, a = iv[b]
        rows = slice(b * bs, (b + 1) * bs)
        for h in range(Hq):
            g = h // G
            keys, vals = _block_keys(k, v, kb, vb, S, a, b, bs, g, block_keys_in_context)
            s = scale * (q[rows, h, :] @ keys.T)              # [bs, n_keys]
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            O[rows, h, :] = (p @ vals) / l
            LSE[rows, h] = (m + np.log(l))[:, 0]
    return O, LSE


def attention_bwd(q, k, v, kb, vb, dout, sample_lens, anchors, block_size: int, scale: float,
                  blocks: Optional[Iterable[int]] = None, block_keys_in_context: bool = False
                  ) -> Dict[str, np.ndarray]:
    """Analytic gradients dq, dk, dv, dkb, dvb (float64) of sum(dout * O).

    Per block b and head h with P = softmax(s) over the allowed keys:
    dvalues = P^T dout; dP = dout values^T; Delta = rowsum(P * dP);
    dS = P * (dP - Delta); dq = scale * dS keys; dkeys = scale * dS^T q.
    Context-key gradients are summed over every (block, head) that reads the key.
    `blocks` restricts the sum to some blocks (then dk/dv are exact only on keys
    that no other block reads).
    """
    Nq, Hq, d = q.shape
    N, Hkv, _ = k.shape
    G = _group(Hq, Hkv)
    bs = int(block_size)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkb = None if block_keys_in_context else np.zeros_like(kb)
    dvb = None if block_keys_in_context else np.zeros_like(vb)
    iv = context_interval(sample_lens, anchors, bs, block_keys_in_context)
    for b in (range(len(iv)) if blocks is None else blocks):
        S, a = iv[b]
        rows = slice(b * bs, (b + 1) * bs)
        n_ctx = a - S
        for h in range(Hq):
            g = h // G
            keys, vals = _block_keys(k, v, kb, vb, S, a, b, bs, g, block_keys_in_context)
            s = scale * (q[rows, h, :] @ keys.T)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            P = p / p.sum(axis=1, keepdims=True)
            dO = dout[rows, h, :]
            dvals = P.T @ dO
            dP = dO @ vals.T
            delta = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - delta)
            dq[rows, h, :] = scale * (dS @ keys)
            dkeys = scale * (dS.T @ q[rows, h, :])
            dk[S:a, g, :] += dkeys[:n_ctx]
            dv[S:a, g, :] += dvals[:n_ctx]
            if not block_keys_in_context:
                dkb[rows, g, :] += dkeys[n_ctx:]
                dvb[rows, g, :] += dvals[n_ctx:]
    return {"dq": dq, "dk": dk, "dv": dv, "dkb": dkb, "dvb": dvb}


def partial(scores: np.ndarray, vals: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(m, l, O) of one row set over one key subset; empty subset -> (-inf, 0, 0)."""
    rows = scores.shape[0]
    if scores.shape[1] == 0:
        return (np.full(rows, NEG_INF), np.zeros(rows), np.zeros((rows, vals.shape[1])))
    m = scores.max(axis=1)
    p = np.exp(scores - m[:, None])
    l = p.sum(axis=1)
    return m, l, (p @ vals) / l[:, None]


def merge(records: List[Tuple[np.ndarray, np.ndarray, np.ndarray]]) -> Tuple[np.ndarray, np.ndarray]:
    """Exact log-sum-exp merge of partial records (m, l, O) over disjoint key subsets."""
    m = np.stack([r[0] for r in records])          # [X, rows]
    l = np.stack([r[1] for r in records])
    O = np.stack([r[2] for r in records])          # [X, rows, d]
    live = l > 0
    M = np.where(live, m, NEG_INF).max(axis=0)     # [rows]
    has = np.isfinite(M)
    Msafe = np.where(has, M, 0.0)
    w = np.where(live, l * np.exp(np.where(live, m, 0.0) - Msafe[None, :]), 0.0)
    L = w.sum(axis=0)
    out = np.zeros(O.shape[1:])
    out[has] = (w[:, has, None] * O[:, has, :]).sum(axis=0) / L[has, None]
    lse = np.full(M.shape, NEG_INF)
    lse[has] = M[has] + np.log(L[has])
    return out, lse


def chunk_partials(q, k, v, sample_lens, anchors, block_size: int, kv_chunk: int, scale: float,
                   block_keys_in_context: bool = False) -> List[Dict]:
    """Per (chunk, block) partial records over the block's keys inside the chunk.

    Returns a list in chunk_entries order of dicts with keys c, b, lo, hi,
    m [bs, Hq], l [bs, Hq], O [bs, Hq, d].
    """
    Nq, Hq, d = q.shape
    Hkv = k.shape[1]
    G = _group(Hq, Hkv)
    bs = int(block_size)
    out = []
    for (c, b, lo, hi) in chunk_entries(sample_lens, anchors, kv_chunk, bs, block_keys_in_context):
        rows = slice(b * bs, (b + 1) * bs)
        m = np.zeros((bs, Hq))
        l = np.zeros((bs, Hq))
        O = np.zeros((bs, Hq, d))
        for h in range(Hq):
            g = h // G
            s = scale * (q[rows, h, :] @ k[lo:hi, g, :].T)
            m[:, h], l[:, h], O[:, h, :] = partial(s, v[lo:hi, g, :])
        out.append({"c": c, "b": b, "lo": lo, "hi": hi, "m": m, "l": l, "O": O})
    return out


def block_partials(q, kb, vb, num_blocks: int, block_size: int, scale: float):
    """In-block partial of every block: m, l [Nq, Hq], O [Nq, Hq, d]."""
    Nq, Hq, d = q.shape
    Hkv = kb.shape[1]
    G = _group(Hq, Hkv)
    bs = int(block_size)
    m = np.zeros((Nq, Hq))
    l = np.zeros((Nq, Hq))
    O = np.zeros((Nq, Hq, d))
    for b in range(num_blocks):
        rows = slice(b * bs, (b + 1) * bs)
        for h in range(Hq):
            g = h // G
            s = scale * (q[rows, h, :] @ kb[rows, g, :].T)
            m[rows, h], l[rows, h], O[rows, h, :] = partial(s, vb[rows, g, :])
    return m, l, O


def split_fwd(q, k, v, kb, vb, sample_lens, anchors, block_size: int, kv_chunk: int, scale: float,
              block_keys_in_context: bool = False):
    """Forward by the split form: chunk partials (+ the in-block partial under reading A), then merge."""
    Nq, Hq, d = q.shape
    bs = int(block_size)
    A = len(anchors)
    parts = chunk_partials(q, k, v, sample_lens, anchors, bs, kv_chunk, scale, block_keys_in_context)
    if not block_keys_in_context:
        bm, bl, bO = block_partials(q, kb, vb, A, bs, scale)
    O = np.zeros((Nq, Hq, d))
    LSE = np.zeros((Nq, Hq))
    for b in range(A):
        rows = slice(b * bs, (b + 1) * bs)
        recs = [] if block_keys_in_context else [(bm[rows].reshape(-1), bl[rows].reshape(-1),
                                                   bO[rows].reshape(-1, d))]
        for p in parts:
            if p["b"] == b:
                recs.append((p["m"].reshape(-1), p["l"].reshape(-1), p["O"].reshape(-1, d)))
        o, lse = merge(recs)
        O[rows] = o.reshape(bs, Hq, d)
        LSE[rows] = lse.reshape(bs, Hq)
    return O, LSE
