"""Barrier protocols of the tcgen05 kernels, checked on randomised schedules (CPU only).

The forward, dK/dV and dQ kernels are warp-specialised: a TMA producer thread, an MMA
issuing thread and element-wise warps hand buffers to one another through mbarriers.
These tests model each kernel's roles as they are written (the waits, arrivals and
commits in program order) and run them under random interleavings, with every role and
engine given a random speed, checking three things:

* every wait starts at most one phase ahead of its barrier and never sees a phase pass
  unobserved (an mbarrier parity wait is only meaningful within that window);
* every buffer -- shared-memory stages, tensor-memory score / output / accumulator
  columns, the Q tile -- holds what its reader expects when it reads it, and is not
  overwritten before its last reader has run;
* every role finishes (no cycle of waits).

MMAs execute in issue order and a commit arrives once every MMA issued before it has
executed (tcgen05.commit); TMA loads land at random times.  Each model is also run with
one wait or one ordering removed, to show that the checks see the hazard it guards.
No GPU is involved; the tests pin the synchronisation design, not the arithmetic.
"""

import random

import pytest


class Bar:
    def __init__(self, count=1):
        self.count, self.k, self.arr = count, 0, 0

    def arrive(self):
        self.arr += 1
        if self.arr == self.count:
            self.arr = 0
            self.k += 1


class Hazard(AssertionError):
    pass


class Core:
    """Barriers, the in-order MMA queue, pending loads and the random scheduler."""

    def __init__(self, seed, names):
        self.rng = random.Random(seed)
        self.B = {n: Bar() for n in names}
        self.mq, self.tma = [], []
        self.speed = {}

    def check(self, cond, msg):
        if not cond:
            raise Hazard(msg)

    def wait(self, bar, n):
        b = self.B[bar]
        self.check(n <= b.k <= n + 1, f"{bar}: waiting for phase {n} with {b.k} complete")
        while b.k < n + 1:
            yield
        self.check(b.k == n + 1, f"{bar}: a phase passed unobserved")

    def mma(self, fn):
        self.mq.append(("mma", fn))

    def commit(self, bar):
        self.mq.append(("commit", bar))

    def load(self, bar, fn):
        self.tma.append((bar, fn))

    def run(self, roles, max_steps=400_000):
        done = set()
        engines = ["<tensor pipe>", "<tma>"]   # not role names
        speed = {r: self.rng.choice([0.05, 0.3, 1.0, 3.0]) for r in list(roles) + engines}
        for _ in range(max_steps):
            if len(done) == len(roles) and not self.mq and not self.tma:
                return
            ch = [r for r in roles if r not in done] + engines
            r = self.rng.choices(ch, [speed[c] for c in ch])[0]
            if r == "<tensor pipe>":
                if self.mq:
                    kind, x = self.mq.pop(0)
                    x() if kind == "mma" else self.B[x].arrive()
            elif r == "<tma>":
                if self.tma:
                    bar, fn = self.tma.pop(self.rng.randrange(len(self.tma)))
                    fn()
                    self.B[bar].arrive()
            else:
                try:
                    next(roles[r])
                except StopIteration:
                    done.add(r)
        raise Hazard(f"no progress (finished: {sorted(done)})")


# ---------------------------------------------------------------------------
# forward kernel: query tiles two at a time (A, B), K and V rings of two stages each (a
# pair's first K/V tiles requested before its Q buffer frees); two softmax warpgroups,
# one per half of the rows of every score tile, take tile A then tile B at each key
# tile; the records leave through separate epilogue warps (the tile's last
# PV and the softmax's row statistics, double-buffered by pair parity, hand each tile
# over; the epilogue releases O after reading it)
# ---------------------------------------------------------------------------
class Forward(Core):
    def __init__(self, pairs, seed, drop=None):
        names = ["q_full", "q_empty", "k_full0", "k_full1", "v_full0", "v_full1", "k_empty0", "k_empty1",
                 "v_empty0", "v_empty1", "s_ready0", "s_ready1", "p_ready0", "p_ready1", "o_ready0", "o_ready1",
                 "o_free0", "o_free1", "o_full0", "o_full1", "stats0_0", "stats0_1", "stats1_0", "stats1_1"]
        super().__init__(seed, names)
        for n in ("p_ready0", "p_ready1", "stats0_0", "stats0_1", "stats1_0", "stats1_1"):
            self.B[n] = Bar(2)        # one arrival per softmax warpgroup
        self.pairs = pairs            # [(nx, n_kt)]
        self.drop = drop
        self.Q = None
        self.K = [None, None]
        self.V = [None, None]
        self.S = [None, None]
        self.O = [None, None]
        self.ST = {}                  # (tile, buffer) -> (pair, halves written) or ("read",)
        self.PH = [set(), set()]      # warpgroups whose rows' P of the current key tile is in S_x
        self.rescale = {}

    def producer(self):
        kv = 0

        def load_kv(c):
            s = c % 2
            if c >= 2 and self.drop != "kv_empty":
                yield from self.wait(f"k_empty{s}", c // 2 - 1)
            self.load(f"k_full{s}", lambda s=s, c=c: self.K.__setitem__(s, c))
            if c >= 2 and self.drop != "kv_empty":
                yield from self.wait(f"v_empty{s}", c // 2 - 1)
            self.load(f"v_full{s}", lambda s=s, c=c: self.V.__setitem__(s, c))
        for i, (nx, nkt) in enumerate(self.pairs):
            yield from load_kv(kv)
            if i >= 1 and self.drop != "q_empty":
                yield from self.wait("q_empty", i - 1)
            self.load("q_full", lambda i=i: setattr(self, "Q", i))
            for j in range(1, nkt):
                yield from load_kv(kv + j)
            kv += nkt
            yield

    def mma_thread(self):
        kv = 0
        p_cnt, of_cnt = [0, 0], [0, 0]
        for i, (nx, nkt) in enumerate(self.pairs):
            yield from self.wait("q_full", i)

            def s_mma(x, c, i=i):
                def ex(x=x, c=c, i=i):
                    self.check(self.Q == i and self.K[c % 2] == c, f"S({x},{c}) reads Q {self.Q} K {self.K[c % 2]}")
                    self.check(self.S[x] is None or self.S[x][0] == "read", f"S({x},{c}) overwrites {self.S[x]}")
                    self.S[x] = ("S", i, c)
                self.mma(ex)
                self.commit(f"s_ready{x}")
            yield from self.wait(f"k_full{kv % 2}", kv // 2)
            for x in range(nx):
                s_mma(x, kv)
            self.commit(f"k_empty{kv % 2}")
            for j in range(nkt):
                c = kv + j
                more = j + 1 < nkt
                for x in range(nx):
                    yield from self.wait(f"p_ready{x}", p_cnt[x])
                    p_cnt[x] += 1
                    if j == 0 and self.drop != "o_free":
                        if of_cnt[x] >= 1:
                            yield from self.wait(f"o_free{x}", of_cnt[x] - 1)
                    if j == 0:
                        of_cnt[x] += 1
                    if x == 0:
                        yield from self.wait(f"v_full{c % 2}", c // 2)

                    def pv(x=x, c=c, j=j, i=i):
                        self.check(self.S[x] == ("S", i, c) and self.PH[x] == {0, 1},
                                   f"PV({x},{c}) reads {self.S[x]} with P halves {self.PH[x]}")
                        self.PH[x] = set()
                        self.check(self.V[c % 2] == c, f"PV({x},{c}) reads V {self.V[c % 2]}")
                        self.S[x] = ("read", i, c)
                        if j == 0:
                            self.check(self.O[x] is None or self.O[x][0] == "stored", f"PV overwrites O {self.O[x]}")
                            self.O[x] = ("acc", i, 1)
                        else:
                            self.check(self.O[x] == ("acc", i, j), f"PV({x},{j}) finds O {self.O[x]}")
                            self.O[x] = ("acc", i, j + 1)
                    self.mma(pv)
                    self.commit(f"o_ready{x}")
                    if not more:
                        self.commit(f"o_full{x}")
                    if x == nx - 1:
                        self.commit(f"v_empty{c % 2}")
                    if more:
                        if x == 0:
                            yield from self.wait(f"k_full{(c + 1) % 2}", (c + 1) // 2)
                        s_mma(x, c + 1)
                        if x == nx - 1:
                            self.commit(f"k_empty{(c + 1) % 2}")
                            if j + 2 == nkt:
                                self.commit("q_empty")
            if nkt == 1:
                self.commit("q_empty")
            kv += nkt
            yield

    def softmax(self, h):
        kv = 0
        s_cnt, o_cnt, st_cnt = [0, 0], [0, 0], [0, 0]
        for i, (nx, nkt) in enumerate(self.pairs):
            for j in range(nkt):
                c = kv + j
                for x in range(nx):
                    yield from self.wait(f"s_ready{x}", s_cnt[x])
                    s_cnt[x] += 1
                    self.check(self.S[x] == ("S", i, c) and h not in self.PH[x],
                               f"softmax half {h} ({x},{c}) finds {self.S[x]}")
                    if j > 0 and self.rng.random() < 0.2:   # the rare rescale of O after PV(j - 1)
                        yield from self.wait(f"o_ready{x}", o_cnt[x] + j - 1)
                        self.check(self.O[x] == ("acc", i, j), f"rescale finds O {self.O[x]}")
                    yield
                    self.PH[x].add(h)
                    self.B[f"p_ready{x}"].arrive()
                    if j == nkt - 1:
                        yield             # the statistics follow the tile's last P
                        b = st_cnt[x] % 2
                        old = self.ST.get((x, b), ("read",))
                        fresh = old == ("read",)
                        self.check(fresh or (old[0] == i and h not in old[1]),
                                   f"stats({x},{b}) of pair {i} overwrite unread {old}")
                        self.ST[(x, b)] = (i, (set() if fresh else old[1]) | {h})
                        self.B[f"stats{x}_{b}"].arrive()
                        st_cnt[x] += 1
            for x in range(nx):
                o_cnt[x] += nkt
            kv += nkt

    def epilogue(self):
        pc = [0, 0]
        for i, (nx, nkt) in enumerate(self.pairs):
            for x in range(nx):
                yield from self.wait(f"o_full{x}", pc[x])
                b = pc[x] % 2
                if self.drop != "stats":
                    yield from self.wait(f"stats{x}_{b}", pc[x] // 2)
                self.check(self.ST.get((x, b)) == (i, {0, 1}), f"epilogue({x}) of pair {i} finds stats "
                           f"{self.ST.get((x, b))}")
                self.ST[(x, b)] = ("read",)
                self.check(self.O[x] == ("acc", i, nkt), f"epilogue({x}) of pair {i} finds {self.O[x]}")
                pc[x] += 1
                yield
                self.O[x] = ("stored", i)
                self.B[f"o_free{x}"].arrive()
                yield

    def go(self):
        self.run({"prod": self.producer(), "mma": self.mma_thread(), "sm0": self.softmax(0), "sm1": self.softmax(1),
                  "epi": self.epilogue()})


# ---------------------------------------------------------------------------
# dK/dV kernel: K, V stationary per key tile, Q / dO double-buffered per pair; within a
# key tile the next pair's S^T is issued right after this pair's dV
# ---------------------------------------------------------------------------
class DKDV(Core):
    def __init__(self, ktiles, seed, drop=None):
        names = ["kv_full", "kv_empty", "qd_full0", "qd_full1", "qd_empty0", "qd_empty1", "st_ready", "dpt_ready",
                 "pt_ready", "dst_ready", "dkv_ready", "dkv_free", "meta_ready0", "meta_ready1", "meta_free0",
                 "meta_free1"]
        super().__init__(seed, names)
        self.kt = ktiles               # pairs (query tiles) meeting each key tile
        self.drop = drop
        self.KV = None
        self.Q = [None, None]
        self.ST, self.DP, self.ACC = None, None, None
        self.META = [None, None]
        self.npairs = sum(ktiles)

    def producer(self):
        q = 0
        for k, n in enumerate(self.kt):
            if k >= 1 and self.drop != "kv_empty":
                yield from self.wait("kv_empty", k - 1)
            self.load("kv_full", lambda k=k: setattr(self, "KV", k))
            for _ in range(n):
                s = q % 2
                if q >= 2 and self.drop != "qd_empty":
                    yield from self.wait(f"qd_empty{s}", q // 2 - 1)
                self.load(f"qd_full{s}", lambda s=s, q=q: self.Q.__setitem__(s, q))
                q += 1
            yield

    def meta(self):
        for q in range(self.npairs):
            m = q % 2
            if q >= 2:
                yield from self.wait(f"meta_free{m}", q // 2 - 1)
            self.META[m] = q
            self.B[f"meta_ready{m}"].arrive()
            yield

    def mma_thread(self):
        q, pds, tiles_done = 0, 0, 0
        for k, n in enumerate(self.kt):
            yield from self.wait("kv_full", k)
            s_issued = False      # S^T of this pair issued ahead, right after the previous dV

            def st_mma(qq, k=k):
                def st(qq=qq, ss=qq % 2, k=k):
                    self.check(self.KV == k and self.Q[ss] == qq, f"S^T({qq}) reads KV {self.KV} Q {self.Q[ss]}")
                    self.check(self.ST is None or self.ST[0] == "read", f"S^T({qq}) overwrites {self.ST}")
                    self.ST = ("S", qq)
                self.mma(st)
                self.commit("st_ready")
            for u in range(n):
                s = q % 2
                if not s_issued:
                    yield from self.wait(f"qd_full{s}", q // 2)
                    st_mma(q)
                s_issued = False

                def dpt(q=q, s=s, k=k):
                    self.check(self.KV == k and self.Q[s] == q, f"dP^T({q}) reads KV {self.KV} Q {self.Q[s]}")
                    self.check(self.DP is None or self.DP[0] == "read", f"dP^T({q}) overwrites {self.DP}")
                    self.DP = ("dP", q)
                self.mma(dpt)
                self.commit("dpt_ready")
                last = u + 1 == n
                if last:
                    self.commit("kv_empty")
                yield from self.wait("pt_ready", pds)
                if u == 0 and tiles_done >= 1 and self.drop != "dkv_free":
                    yield from self.wait("dkv_free", tiles_done - 1)

                def dv(q=q, s=s, u=u, k=k):
                    self.check(self.ST == ("P", q) and self.Q[s] == q, f"dV({q}) reads {self.ST}")
                    if u == 0:
                        self.check(self.ACC is None or self.ACC[0] == "stored", f"dV overwrites {self.ACC}")
                        self.ACC = ("acc", k, 0)
                    self.ST = ("read", q)
                if not last and self.drop == "lookahead_before_dv":
                    yield from self.wait(f"qd_full{(q + 1) % 2}", (q + 1) // 2)
                    st_mma(q + 1)
                    s_issued = True
                self.mma(dv)
                if not last and self.drop != "lookahead_before_dv":
                    # the next pair's S^T right behind dV, its P^T's last reader
                    yield from self.wait(f"qd_full{(q + 1) % 2}", (q + 1) // 2)
                    st_mma(q + 1)
                    s_issued = True
                yield from self.wait("dst_ready", pds)
                pds += 1

                def dk(q=q, s=s, u=u, k=k):
                    self.check(self.DP == ("dS", q) and self.Q[s] == q, f"dK({q}) reads {self.DP}")
                    self.check(self.ACC == ("acc", k, u), f"dK({q}) finds {self.ACC}")
                    self.ACC = ("acc", k, u + 1)
                    self.DP = ("read", q)
                self.mma(dk)
                self.commit(f"qd_empty{s}")
                q += 1
            if n > 0:
                self.commit("dkv_ready")
                tiles_done += 1
            else:
                self.commit("kv_empty")
            yield

    def elementwise(self):
        q, tiles_done = 0, 0
        for k, n in enumerate(self.kt):
            for _ in range(n):
                m = q % 2
                yield from self.wait(f"meta_ready{m}", q // 2)
                self.check(self.META[m] == q, "metadata of another pair")
                yield from self.wait("st_ready", q)
                self.check(self.ST == ("S", q), f"P^T pass {q} finds {self.ST}")
                yield
                self.ST = ("P", q)
                self.B["pt_ready"].arrive()
                yield from self.wait("dpt_ready", q)
                self.check(self.DP == ("dP", q), f"dS^T pass {q} finds {self.DP}")
                yield
                self.DP = ("dS", q)
                self.B["dst_ready"].arrive()
                self.B[f"meta_free{m}"].arrive()
                q += 1
            if n > 0:
                yield from self.wait("dkv_ready", tiles_done)
                self.check(self.ACC == ("acc", k, n), f"epilogue of key tile {k} finds {self.ACC}")
                yield
                self.ACC = ("stored", k)
                self.B["dkv_free"].arrive()
                tiles_done += 1

    def go(self):
        self.run({"prod": self.producer(), "mma": self.mma_thread(), "ew": self.elementwise(), "meta": self.meta()})


# ---------------------------------------------------------------------------
# dQ kernel: Q / dO per query tile; a K ring of three stages (released after dQ += dS K)
# and one V stage (released once dP has read it), K loaded before V; a tile's first K/V
# before its Q / dO; S double-buffered; the next dP issued before dQ; dQ read and
# released by epilogue warps of its own
# ---------------------------------------------------------------------------
class DQ(Core):
    def __init__(self, tiles, seed, drop=None):
        names = ["qd_full", "qd_empty", "k_full0", "k_full1", "k_full2", "v_full", "k_empty0", "k_empty1",
                 "k_empty2", "v_empty", "s_ready0", "s_ready1", "dp_ready", "ds_ready", "dq_ready", "dq_free",
                 "meta_ready0", "meta_ready1", "meta_free0", "meta_free1"]
        super().__init__(seed, names)
        self.tiles = tiles
        self.drop = drop
        self.QD = None
        self.K, self.V, self.S = [None, None, None], [None], [None, None]
        self.DP, self.DQ = None, None
        self.META = [None, None]

    def producer(self):
        kv = 0

        def load_kv(c):   # K: a ring of three stages; V: one stage
            s = c % 3
            if c >= 3 and self.drop != "kv_empty":
                yield from self.wait(f"k_empty{s}", c // 3 - 1)
            self.load(f"k_full{s}", lambda s=s, c=c: self.K.__setitem__(s, c))
            if c >= 1 and self.drop != "v_empty":
                yield from self.wait("v_empty", c - 1)
            self.load("v_full", lambda c=c: self.V.__setitem__(0, c))
        for n, nkt in enumerate(self.tiles):
            yield from load_kv(kv)
            if n >= 1 and self.drop != "qd_empty":
                yield from self.wait("qd_empty", n - 1)
            self.load("qd_full", lambda n=n: setattr(self, "QD", n))
            for j in range(1, nkt):
                yield from load_kv(kv + j)
            kv += nkt
            yield

    def meta(self):
        for n in range(len(self.tiles)):
            m = n % 2
            if n >= 2:
                yield from self.wait(f"meta_free{m}", n // 2 - 1)
            self.META[m] = n
            self.B[f"meta_ready{m}"].arrive()
            yield

    def mma_thread(self):
        kv, ds = 0, 0
        for n, nkt in enumerate(self.tiles):
            yield from self.wait("qd_full", n)

            def s_mma(c, n=n):
                def ex(b=c % 2, c=c, n=n):
                    self.check(self.QD == n and self.K[c % 3] == c, f"S({c}) reads QD {self.QD} K {self.K[c % 3]}")
                    self.check(self.S[b] is None or self.S[b][0] == "read", f"S({c}) overwrites {self.S[b]}")
                    self.S[b] = ("S", c)
                self.mma(ex)
                self.commit(f"s_ready{c % 2}")

            def dp_mma(c, n=n):
                def ex(c=c, n=n):
                    self.check(self.QD == n and self.V[0] == c, f"dP({c}) reads QD {self.QD} V {self.V[0]}")
                    self.check(self.DP is None or self.DP[0] == "read", f"dP({c}) overwrites {self.DP}")
                    self.DP = ("dP", c)
                self.mma(ex)
                self.commit("dp_ready")
                self.commit("v_empty")
            c0 = kv
            yield from self.wait(f"k_full{c0 % 3}", c0 // 3)
            s_mma(c0)
            yield from self.wait("v_full", c0)
            dp_mma(c0)
            for j in range(nkt):
                c = c0 + j
                more = j + 1 < nkt
                if more:
                    yield from self.wait(f"k_full{(c + 1) % 3}", (c + 1) // 3)
                    s_mma(c + 1)
                yield from self.wait("ds_ready", ds)
                ds += 1
                if more:
                    yield from self.wait("v_full", c + 1)
                    dp_mma(c + 1)
                    if j + 2 == nkt:
                        self.commit("qd_empty")
                if j == 0 and n >= 1 and self.drop != "dq_free":
                    yield from self.wait("dq_free", n - 1)

                def dq(b=c % 2, c=c, j=j, n=n):
                    self.check(self.S[b] == ("dS", c) and self.K[c % 3] == c,
                               f"dQ({c}) reads {self.S[b]} K {self.K[c % 3]}")
                    if j == 0:
                        self.check(self.DQ is None or self.DQ[0] == "stored", f"dQ overwrites {self.DQ}")
                        self.DQ = ("acc", n, 1)
                    else:
                        self.check(self.DQ == ("acc", n, j), f"dQ({j}) finds {self.DQ}")
                        self.DQ = ("acc", n, j + 1)
                    self.S[b] = ("read", c)
                self.mma(dq)
                self.commit(f"k_empty{c % 3}")
            self.commit("dq_ready")
            if nkt == 1:
                self.commit("qd_empty")
            kv += nkt
            yield

    def elementwise(self):
        kv = 0
        for n, nkt in enumerate(self.tiles):
            m = n % 2
            yield from self.wait(f"meta_ready{m}", n // 2)
            self.check(self.META[m] == n, "metadata of another tile")
            self.B[f"meta_free{m}"].arrive()
            for j in range(nkt):
                c = kv + j
                yield from self.wait(f"s_ready{c % 2}", c // 2)
                yield from self.wait("dp_ready", c)
                self.check(self.S[c % 2] == ("S", c), f"element-wise {c} finds S {self.S[c % 2]}")
                self.check(self.DP == ("dP", c), f"element-wise {c} finds dP {self.DP}")
                yield
                self.S[c % 2] = ("dS", c)
                self.DP = ("read", c)
                self.B["ds_ready"].arrive()
            kv += nkt

    def epilogue(self):   # warps of its own: reads dQ, releases it, then stores
        for n, nkt in enumerate(self.tiles):
            yield from self.wait("dq_ready", n)
            self.check(self.DQ == ("acc", n, nkt), f"epilogue {n} finds {self.DQ}")
            yield
            self.DQ = ("stored", n)
            self.B["dq_free"].arrive()

    def go(self):
        self.run({"prod": self.producer(), "mma": self.mma_thread(), "ew": self.elementwise(), "meta": self.meta(),
                  "epi": self.epilogue()})


# ---------------------------------------------------------------------------
# dq reduce kernel: the block role computes the in-block dq of 32 rows at a time into one
# of two shared-memory slots and arrives on the slot's "full" named barrier; the stream
# role sums the rows' chunk partials, syncs on "full", adds the slot, and arrives on the
# slot's "empty" barrier when the block role will write that slot again (pass j + 2);
# the block role syncs on "empty" before its third and later passes.  A named barrier
# (bar.sync / bar.arrive with a count of both roles' threads) completes a phase at every
# second group arrival, whoever makes it.
# ---------------------------------------------------------------------------
class NamedBar:
    def __init__(self):
        self.arr, self.phase = 0, 0

    def arrive(self):
        ph = self.phase
        self.arr += 1
        if self.arr == 2:
            self.arr = 0
            self.phase += 1
        return ph


class Reduce(Core):
    def __init__(self, npass, seed, drop=None):
        super().__init__(seed, [])
        self.npass, self.drop = npass, drop
        self.N = {f"{k}{s}": NamedBar() for k in ("full", "empty") for s in (0, 1)}
        self.slot = [None, None]   # pass whose in-block dq the slot holds (None: consumed)

    def sync(self, name):
        ph = self.N[name].arrive()
        while self.N[name].phase <= ph:
            yield

    def stream(self):
        for j in range(self.npass):
            for _ in range(self.rng.randint(1, 4)):   # the chunk partials of the rows
                yield
            sl = j & 1
            yield from self.sync(f"full{sl}")
            self.check(self.slot[sl] == j, f"stream pass {j} read slot {sl} holding {self.slot[sl]}")
            self.slot[sl] = None
            if j + 2 < self.npass:
                self.N[f"empty{sl}"].arrive()
            yield

    def block(self):
        for j in range(self.npass):
            for _ in range(self.rng.randint(1, 3)):   # P, dS and the in-block dq of the rows
                yield
            sl = j & 1
            if j >= 2 and self.drop != "empty":
                yield from self.sync(f"empty{sl}")
            self.check(self.slot[sl] is None, f"block pass {j} overwrote slot {sl} holding {self.slot[sl]}")
            self.slot[sl] = j
            self.N[f"full{sl}"].arrive()
            yield
        for _ in range(self.rng.randint(0, 3)):   # dkb, dvb
            yield

    def go(self):
        self.run({"stream": self.stream(), "block": self.block()})
        self.check(all(b.arr == 0 for b in self.N.values()), "a named barrier left with a pending arrival")


# ---------------------------------------------------------------------------
def _fwd_case(rng, seed, drop=None):
    pairs = [(rng.choice([1, 2, 2]), rng.choice([1, 1, 2, 3, 4, 6])) for _ in range(rng.randint(1, 12))]
    return Forward(pairs, seed, drop)


def _dkdv_case(rng, seed, drop=None):
    return DKDV([rng.choice([0, 1, 1, 2, 3, 4, 6]) for _ in range(rng.randint(1, 12))], seed, drop)


def _dq_case(rng, seed, drop=None):
    return DQ([rng.choice([1, 1, 2, 3, 4, 6]) for _ in range(rng.randint(1, 12))], seed, drop)


def _reduce_case(rng, seed, drop=None):
    return Reduce(rng.randint(1, 6), seed, drop)


CASES = {"forward": _fwd_case, "dkdv": _dkdv_case, "dq": _dq_case, "reduce": _reduce_case}


@pytest.mark.parametrize("kernel", list(CASES))
def test_protocol_holds_on_random_schedules(kernel):
    rng = random.Random(11)
    for seed in range(400):
        CASES[kernel](rng, seed).go()


@pytest.mark.parametrize("kernel,drop", [("forward", "kv_empty"), ("forward", "q_empty"), ("forward", "o_free"),
                                         ("forward", "stats"),
                                         ("dkdv", "qd_empty"),
                                         ("dkdv", "kv_empty"), ("dkdv", "lookahead_before_dv"),
                                         ("dq", "kv_empty"), ("dq", "v_empty"), ("dq", "dq_free"),
                                         ("reduce", "empty")])
def test_each_producer_guard_is_needed(kernel, drop):
    """Removing one of the producer's waits lets some schedule overwrite a stage that an
    MMA has not read yet; issuing the dK/dV kernel's look-ahead S^T before dV instead of
    after it overwrites a P^T that dV has not read; without the forward MMA's wait for the
    epilogue warps to release O, the next pair's first PV overwrites an O not yet read (and
    likewise the dQ kernel's next tile's first dQ += dS K)."""
    rng = random.Random(5)
    caught = 0
    for seed in range(300):
        try:
            CASES[kernel](rng, seed, drop).go()
        except Hazard:
            caught += 1
            break
    assert caught > 0


@pytest.mark.parametrize("kernel,drop", [("dkdv", "dkv_free"), ("dq", "qd_empty")])
def test_guard_is_implied_by_program_order(kernel, drop):
    """Some waits are redundant, kept as guards; these schedules show that nothing depends
    on them.  In the dK/dV kernel the MMA thread's wait for the epilogue to release the
    accumulators: the epilogue runs on the element-wise warps before their next pass, which
    the first product into an accumulator already waits for.  (The forward's and the dQ
    kernel's epilogues run on warps of their own, so there the wait is needed: see above.)
    In the dQ kernel the
    producer's wait for the Q / dO buffer: it loads a tile's Q / dO only after the single
    V stage was released by the previous tile's last dP, which the tensor pipe executes
    after the last products reading Q / dO."""
    rng = random.Random(6)
    for seed in range(150):
        CASES[kernel](rng, seed, drop).go()
