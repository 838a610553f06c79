"""A model of the tensor-core prefill attention kernel's barrier protocol, run under random schedules.

The kernel (chunk_wise_hierarchical_hils_b200/csrc/attend_prefill_tc.cu) coordinates its roles with
mbarriers only: a key loader and a value loader (TMA copies into rings of shared-memory slots), a key
product issuer and a value product issuer (tcgen05.mma into TMEM), and twelve softmax warps in three
groups (chunk t goes to group t % 3).  Here every role is a generator that yields the condition it
waits on; a scheduler runs a random runnable role at each step, and copies and MMAs complete after
random delays (one issuer's MMAs in issue order).  An mbarrier is modelled by its phase count, pending
arrivals and pending transaction bytes, and a parity wait behaves as the hardware's does: it succeeds
when the barrier's current phase parity differs from the waited parity, so a waiter more than one
phase behind aliases.

Buffer states are tracked alongside and every access is checked: a key or value slot is not
overwritten before its product read it, an S buffer not before its eight softmax warps read it, a P
buffer not before its value product read it, O not before the epilogue read it, Q not before its
tile's key products finished, and the tile bookkeeping not while a role still reads it.  A run that
violates one of them, or stops with no role able to move, fails.

`tiles` lists the chunk-union sizes of the query tiles one CTA processes: one entry is the kernel as
built (one tile per CTA); several entries model a persistent CTA that walks tiles back to back with
double-buffered bookkeeping and an O_EMPTY barrier.
"""
import random


class _Version:
    n = 0


class Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.phase = 0          # completed phases
        self.pending = count
        self.tx = 0

    def _moved(self):
        _Version.n += 1
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, n=1):
        self.pending -= n
        if self.pending < 0:
            raise AssertionError("%s: more arrivals than its count" % self.name)
        self._moved()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        if self.tx < 0:
            raise AssertionError("%s: transaction count below zero" % self.name)
        self._moved()

    def done(self, parity):
        return (self.phase & 1) != parity


class Protocol:
    """p_mod_2: P buffers and their PV_READY / PV_DONE barriers go by pair % 2 (the kernel as built);
    False ties them to the value slots (pair % n_value_slots), the earlier design.
    lone_by_count: the four warps of a lone last chunk arrive with count 2 (needed once a tile
    follows); False lets the value loader stand in with four extra arrivals (enough for one tile)."""

    def __init__(self, tiles, n_value_slots, seed=0, p_mod_2=True, lone_by_count=None):
        self.r = random.Random(seed)
        self.tiles = list(tiles)
        self.NSV = n_value_slots
        self.NP = 2 if p_mod_2 else n_value_slots
        self.lone_by_count = (len(self.tiles) > 1) if lone_by_count is None else lone_by_count
        self.events = []
        self.mma_queues = {}
        self.now = 0
        self.B = {}
        self._bar("Q_FULL", 1)
        for s in range(2):
            self._bar("K_LAND%d" % s, 1)
            self._bar("QK_READY%d" % s, 9)
            self._bar("QK_DONE%d" % s, 1)
            for _ in range(8):
                self.B["QK_READY%d" % s].arrive()      # S buffers start free
        for s in range(self.NSV):
            self._bar("V_LAND%d" % s, 1)
        for s in range(self.NP):
            self._bar("PV_READY%d" % s, 9)
            self._bar("PV_DONE%d" % s, 1)
        self._bar("O_FULL", 1)
        self._bar("O_EMPTY", 12)
        self._bar("BOOK0", 1)
        self._bar("BOOK1", 1)
        self.kslot = {s: None for s in range(2)}
        self.vslot = {s: None for s in range(self.NSV)}
        self.s_buf = {s: None for s in range(2)}
        self.s_reads = {s: 0 for s in range(2)}
        self.p_buf = {s: set() for s in range(self.NP)}
        self.o_tile = None
        self.o_unread = None
        self.o_reads = 0
        self.q_state = None
        self.book = {0: None, 1: None}
        self.book_readers = {0: set(), 1: set()}
        self.qk_done = set()
        self.pv_done = set()
        self.out = []

    def _bar(self, name, count):
        self.B[name] = Bar(name, count)

    # -- asynchronous completions
    def _later(self, fn):
        self.events.append((self.now + self.r.randint(1, 30), self.r.random(), fn))

    def _copy(self, bar, nbytes, on_land):
        def land():
            on_land()
            self.B[bar].complete_tx(nbytes)
        self._later(land)

    def _mma(self, issuer, on_done):
        q = self.mma_queues.setdefault(issuer, [])
        q.append(on_done)
        self._later(lambda: q.pop(0)())

    def _moved(self):
        v = _Version.n
        return lambda: _Version.n != v

    def _pairs(self, i):
        return (self.tiles[i] + 1) // 2

    # -- roles
    def key_loader(self):
        base = 0
        for i in range(len(self.tiles)):
            bk = i & 1
            yield lambda: self.B["BOOK%d" % bk].done((i >> 1) & 1)
            assert self.book[bk] == i, "key loader reads another tile's bookkeeping"
            self.book_readers[bk].add("keys")
            if base > 0:
                last = base - 1
                yield lambda: self.B["QK_DONE%d" % (last & 1)].done((last >> 1) & 1)
            assert self.q_state is None or self.q_state[1] == "consumed", "Q overwritten before its products"
            self.B["Q_FULL"].expect_tx(1)
            self.q_state = (i, "loading")
            self._copy("Q_FULL", 1, lambda i=i: setattr(self, "q_state", (i, "landed")))
            n = self._pairs(i)
            issued = landed = 0
            while landed < n:
                g = base + issued
                freed = g - 2
                if issued < n and issued < landed + 2 and (
                        freed < 0 or self.B["QK_DONE%d" % (freed & 1)].done((freed >> 1) & 1)):
                    s = g & 1
                    assert self.kslot[s] is None, "key slot overwritten before its product"
                    self.kslot[s] = ("loading", g)
                    self.B["K_LAND%d" % s].expect_tx(1)
                    self._copy("K_LAND%d" % s, 1, lambda s=s, g=g: self.kslot.__setitem__(s, ("landed", g)))
                    issued += 1
                    continue
                gl = base + landed
                if landed < issued and self.B["K_LAND%d" % (gl & 1)].done((gl >> 1) & 1):
                    self.B["QK_READY%d" % (gl & 1)].arrive()
                    landed += 1
                    continue
                yield self._moved()
            self.book_readers[bk].discard("keys")
            base += n

    def value_loader(self):
        base = 0
        for i in range(len(self.tiles)):
            bk = i & 1
            yield lambda: self.B["BOOK%d" % bk].done((i >> 1) & 1)
            assert self.book[bk] == i, "value loader reads another tile's bookkeeping"
            self.book_readers[bk].add("values")
            n = self._pairs(i)
            issued = landed = 0
            while landed < n:
                g = base + issued
                freed = g - self.NSV
                if issued < n and issued < landed + self.NSV and (
                        freed < 0 or self.B["PV_DONE%d" % (freed % self.NP)].done((freed // self.NP) & 1)):
                    s = g % self.NSV
                    assert self.vslot[s] is None, "value slot overwritten before its product"
                    self.vslot[s] = ("loading", g)
                    self.B["V_LAND%d" % s].expect_tx(1)
                    self._copy("V_LAND%d" % s, 1, lambda s=s, g=g: self.vslot.__setitem__(s, ("landed", g)))
                    issued += 1
                    continue
                gl = base + landed
                if landed < issued and self.B["V_LAND%d" % (gl % self.NSV)].done((gl // self.NSV) & 1):
                    extra = 4 if (not self.lone_by_count and landed == n - 1 and self.tiles[i] & 1) else 0
                    self.B["PV_READY%d" % (gl % self.NP)].arrive(1 + extra)
                    landed += 1
                    continue
                yield self._moved()
            self.book_readers[bk].discard("values")
            base += n

    def key_issuer(self):
        base = 0
        for i in range(len(self.tiles)):
            bk = i & 1
            yield lambda: self.B["BOOK%d" % bk].done((i >> 1) & 1)
            yield lambda: self.B["Q_FULL"].done(i & 1)
            assert self.q_state == (i, "landed"), "key product before its Q landed"
            n = self._pairs(i)
            for j in range(n):
                g = base + j
                s = g & 1
                yield lambda: self.B["QK_READY%d" % s].done((g >> 1) & 1)
                assert self.kslot[s] == ("landed", g), "key product reads a slot that does not hold its pair"
                assert self.s_buf[s] is None, "S buffer overwritten before its softmax warps read it"

                def done(s=s, g=g, last=(j == n - 1), i=i):
                    self.s_buf[s], self.s_reads[s], self.kslot[s] = g, 0, None
                    self.qk_done.add(g)
                    if last:
                        self.q_state = (i, "consumed")
                    self.B["QK_DONE%d" % s].arrive()
                self._mma("keys", done)
                yield None
            base += n

    def value_issuer(self):
        base = 0
        for i in range(len(self.tiles)):
            bk = i & 1
            yield lambda: self.B["BOOK%d" % bk].done((i >> 1) & 1)
            n = self._pairs(i)
            for j in range(n):
                g = base + j
                if j == 0 and i > 0:
                    yield lambda: self.B["O_EMPTY"].done((i - 1) & 1)
                    assert self.o_unread is None, "O overwritten before the epilogue read it"
                if j == 0:
                    self.o_tile = i
                yield lambda: self.B["PV_READY%d" % (g % self.NP)].done((g // self.NP) & 1)
                halves = 2 if 2 * j + 1 < self.tiles[i] else 1
                assert self.vslot[g % self.NSV] == ("landed", g), "value product reads a slot without its pair"
                pb = self.p_buf[g % self.NP]
                assert len(pb) == halves and all(x[0] == g for x in pb), "value product reads an incomplete P"

                def done(g=g):
                    self.vslot[g % self.NSV] = None
                    self.p_buf[g % self.NP] = set()
                    self.pv_done.add(g)
                    self.B["PV_DONE%d" % (g % self.NP)].arrive()
                self._mma("values", done)
                yield None

            def full(i=i):
                self.o_unread = i
                self.B["O_FULL"].arrive()
            self._mma("values", full)
            base += n

    def softmax_warp(self, w):
        grp = w // 4
        base = 0
        yield ("named_barrier", 0)
        if w == 0:
            self.book[0] = 0
            self.B["BOOK0"].arrive()
        for i in range(len(self.tiles)):
            nu = self.tiles[i]
            for t in range(grp, nu, 3):
                g = base + (t >> 1)
                sb, pb = g & 1, g % self.NP
                lone = (t == nu - 1) and (nu & 1)
                yield lambda: self.B["QK_DONE%d" % sb].done((g >> 1) & 1)
                assert self.s_buf[sb] == g, "softmax reads an S buffer that does not hold its pair"
                self.s_reads[sb] += 2 if lone else 1
                if self.s_reads[sb] == 8:
                    self.s_buf[sb] = None
                self.B["QK_READY%d" % sb].arrive(2 if (lone and self.lone_by_count) else 1)
                yield None
                if g >= self.NP:
                    yield lambda: self.B["PV_DONE%d" % pb].done(((g // self.NP) - 1) & 1)
                assert all(x[0] == g for x in self.p_buf[pb]), "P buffer overwritten before its value product"
                if w % 4 == 0:
                    self.p_buf[pb].add((g, t & 1))
                self.B["PV_READY%d" % pb].arrive(2 if (lone and self.lone_by_count) else 1)
                yield None
            base += self._pairs(i)
            if i + 1 < len(self.tiles):
                yield ("named_barrier", 2 * i + 1)
                bk = (i + 1) & 1
                if w == 0:
                    assert not self.book_readers[bk], "bookkeeping rebuilt while a loader reads it"
                    self.book[bk] = i + 1
                yield ("named_barrier", 2 * i + 2)
                if w == 0:
                    self.B["BOOK%d" % bk].arrive()
            yield lambda: self.B["O_FULL"].done(i & 1)
            assert self.o_unread == i and self.o_tile == i, "epilogue reads an O that is not its tile's"
            if w == 0:
                self.out.append(i)
            self.o_reads += 1
            if self.o_reads % 12 == 0:
                self.o_unread = None
            self.B["O_EMPTY"].arrive()
            yield None

    # -- scheduler
    def run(self, max_steps=200000):
        roles = {"keys": self.key_loader(), "values": self.value_loader(), "qk": self.key_issuer(),
                 "pv": self.value_issuer()}
        for w in range(12):
            roles["softmax%d" % w] = self.softmax_warp(w)
        waiting = dict.fromkeys(roles)
        at_barrier = {}
        finished = set()
        for _ in range(max_steps):
            if len(finished) == len(roles):
                break
            runnable = [k for k in roles if k not in finished and k not in at_barrier
                        and (waiting[k] is None or waiting[k]())]
            for bid in set(at_barrier.values()):
                members = [k for k, b in at_barrier.items() if b == bid]
                if len(members) == 12:
                    for k in members:
                        del at_barrier[k]
                        waiting[k] = None
                        runnable.append(k)
            if self.events and (not runnable or self.r.random() < 0.3):
                self.events.sort(key=lambda e: (e[0], e[1]))
                t, _, fn = self.events.pop(self.r.randrange(min(3, len(self.events))))
                self.now = max(self.now, t)
                fn()
                continue
            if not runnable:
                raise AssertionError("deadlock: %s" % sorted(k for k in roles if k not in finished))
            k = self.r.choice(runnable)
            self.now += 1
            try:
                c = next(roles[k])
            except StopIteration:
                finished.add(k)
                continue
            if isinstance(c, tuple):
                at_barrier[k] = c[1]
            else:
                waiting[k] = c
        else:
            raise AssertionError("no completion within the step limit")
        assert self.out == list(range(len(self.tiles))), "tiles finished out of order or missing"
