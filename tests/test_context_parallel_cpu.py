"""Split-KV over ranks, host logic on CPU: gloo ranks (world size 2 and 3) run
SplitKVContextParallel -- rank plans, the query-side broadcasts, the all-to-all
of result rows to their owners -- with the oracle standing in for each rank's
GPU steps (a rank's exact partial result and backward share over the keys its
plan owns, the combine, the sum).  Every rank's outputs must equal the unsplit
oracle on its rows (dk, dv: on its chunks, zero elsewhere).  Context rows of
other ranks' chunks hold NaN on every rank, so any read of them would show.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

LENS = (41, 17, 66, 30)
BS, HQ, HKV, D, C = 4, 4, 2, 8, 13
SCALE = 0.3


def _inputs(A):
    rng = np.random.default_rng(11)
    N = sum(LENS)
    anchors = np.sort(rng.choice(N, size=A, replace=False)).astype(np.int32)
    Nq = A * BS
    t = {n: rng.standard_normal(s) for n, s in (("q", (Nq, HQ, D)), ("k", (N, HKV, D)), ("v", (N, HKV, D)),
                                                ("kb", (Nq, HKV, D)), ("vb", (Nq, HKV, D)), ("dout", (Nq, HQ, D)))}
    return anchors, t


class OracleOps:
    """A rank's local steps by the oracle (float64, CPU)."""

    def __init__(self, cp, anchors, rb):
        self.cp, self.anchors, self.rb = cp, anchors, rb

    def _args(self):
        return (LENS, self.anchors, BS, C, SCALE, self.cp.chunk_owner, self.cp.rank, self.cp.R)

    def local_fwd(self, q, k, v, kb, vb, scale):
        import torch
        from oracle import context_parallel as ocp
        kbn = None if kb is None else kb.numpy()
        vbn = None if vb is None else vb.numpy()
        o, lse = ocp.rank_fwd(q.numpy(), k.numpy(), v.numpy(), kbn, vbn, *self._args(),
                              block_keys_in_context=self.rb)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def combine(self, o_parts, lse_parts, out_dtype):
        import torch
        from oracle import context_parallel as ocp
        o, lse = ocp.combine_ranks(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o), torch.from_numpy(lse)

    def local_bwd(self, q, k, v, kb, vb, o, lse, dout, scale):
        import torch
        from oracle import context_parallel as ocp
        kbn = None if kb is None else kb.numpy()
        vbn = None if vb is None else vb.numpy()
        g = ocp.rank_bwd(q.numpy(), k.numpy(), v.numpy(), kbn, vbn, dout.numpy(), o.numpy(), lse.numpy(),
                         *self._args(), block_keys_in_context=self.rb)
        return {n: None if x is None else torch.from_numpy(x) for n, x in g.items()}

    def sum(self, parts):
        return parts.sum(dim=0)


def _worker(rank, world, port, rb, A, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from context_block_sparse_b200.context_parallel import SplitKVContextParallel
        from oracle import attention as att
        anchors, t = _inputs(A)
        cp = SplitKVContextParallel(LENS, anchors, BS, HQ, HKV, D, C, num_workers=4, block_keys_in_context=rb,
                                    ops=lambda cp: OracleOps(cp, anchors, rb))
        rows = cp.rows
        k, v = t["k"].copy(), t["v"].copy()
        mine = np.zeros(sum(LENS), dtype=bool)
        for lo, hi in cp.owned_rows():
            mine[lo:hi] = True
        k[~mine] = np.nan
        v[~mine] = np.nan
        T = torch.from_numpy
        kb = None if rb else T(t["kb"][rows].copy())
        vb = None if rb else T(t["vb"][rows].copy())
        for _ in range(2):      # a second step reuses the exchange buffers of the first
            o, lse = cp.forward(T(t["q"][rows].copy()), T(k), T(v), kb, vb, SCALE)
            g = cp.backward(T(k), T(v), o, lse, T(t["dout"][rows].copy()), SCALE)
        kbf = None if rb else t["kb"]
        vbf = None if rb else t["vb"]
        O, L = att.attention_fwd(t["q"], t["k"], t["v"], kbf, vbf, LENS, anchors, BS, SCALE,
                                 block_keys_in_context=rb)
        ref = att.attention_bwd(t["q"], t["k"], t["v"], kbf, vbf, t["dout"], LENS, anchors, BS, SCALE,
                                block_keys_in_context=rb)
        def mx(a, b=0.0):
            d = np.abs(a - b)
            return float(d.max()) if d.size else 0.0

        err = {
            "o": mx(o.numpy(), O[rows]),
            "lse": mx(lse.numpy(), L[rows]),
            "dq": mx(g["dq"].numpy(), ref["dq"][rows]),
            "dk": mx(g["dk"].numpy()[mine], ref["dk"][mine]),
            "dv": mx(g["dv"].numpy()[mine], ref["dv"][mine]),
            "dk_elsewhere": mx(g["dk"].numpy()[~mine]),
            "shape": 0.0 if o.shape[0] == rows.stop - rows.start else 1.0,
        }
        if not rb:
            err["dkb"] = mx(g["dkb"].numpy(), ref["dkb"][rows])
            err["dvb"] = mx(g["dvb"].numpy(), ref["dvb"][rows])
        q.put((rank, cp.block_range, int(mine.sum()), err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,rb,A", [(2, False, 7), (3, False, 7), (2, True, 7), (3, False, 2)])
def test_gloo_ranks_reproduce_unsplit_attention(world, rb, A):
    """(3 ranks, 2 blocks: rank 0 holds no query rows and takes part in every exchange.)"""
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rb, A, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # block ranges tile [0, A), owned context rows tile [0, N)
    assert [o[1] for o in out] == [((r * A) // world, ((r + 1) * A) // world) for r in range(world)]
    assert sum(o[2] for o in out) == sum(LENS)
    for rank, _, _, err in out:
        for n, e in err.items():
            assert e < 1e-12, (rank, n, e)
