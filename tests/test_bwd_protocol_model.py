"""Model check of the backward kernels' synchronisation protocol (no GPU).

compute-sanitizer is not available for these kernels, so the protocol they
follow -- mbarrier phases, the ring of streamed 64-row tiles, the two TMEM
buffers of S and dP, the separate commits of S and dP, and the in-order
tensor pipe -- is restated here as a small discrete-event model and run under
many random interleavings of the warps, the TMA engine and the tensor pipe.
The model checks, at every step:

- a parity wait only succeeds on the phase it means (never one phase early,
  never aliased two phases late);
- a TMA copy never lands in a ring slot an issued, unfinished product still
  reads, and every product reads the tiles of its own step;
- the elementwise warps read S (and dP) of a buffer only after the products
  that write them completed, and only while they hold their own step;
- a product that overwrites S or dP of a buffer never runs before the
  accumulating product that reads P or dS from it, and the accumulating
  products read P/dS only after every elementwise warp wrote them;
- the per-step statistics in a ring slot are not rewritten while a warp still
  reads them;
- every role finishes (no deadlock) and nothing is in flight at exit.

Planted mistakes (a copy issued before its slot is free, a wrong parity, the
next S issued before the product that reads the buffer) must be caught, so the
model is known to be able to fail.  Each role mirrors the warp of the same name
in csrc/sdpa_bwd_pipe_sm100.cuh.
"""
import random

import pytest


class ModelError(AssertionError):
    pass


def check(cond, *what):
    if not cond:
        raise ModelError(what)


class Bar:
    """mbarrier: `count` arrivals plus expected transaction bytes complete a
    phase; try_wait.parity(P) succeeds iff the phase count's parity != P."""

    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, 0, 0, 0

    def arrive(self, tx=0):
        self.pending += 1
        self.tx += tx
        self._maybe_complete()

    def complete_tx(self, n):
        self.tx -= n
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == self.count and self.tx == 0:
            self.pending, self.phase = 0, self.phase + 1

    def ready(self, parity, intended):
        """The wait for completion number `intended` (0-based) with `parity`."""
        if (self.phase & 1) == parity:
            return False
        check(self.phase == intended + 1, "phase aliasing", self.name, self.phase, intended)
        return True


class Machine:
    def __init__(self, seed, n_warps=8):
        self.rng = random.Random(seed)
        self.tma = []                  # (bar, buffer, step)
        self.pipe = []                 # in-order: ("mma", fn) or ("commit", bar)
        self.buf = {}                  # buffer -> step it holds (None while loading)
        self.readers = {}              # buffer -> issued, unfinished MMAs reading it
        self.n_warps = n_warps
        self.cta_arrived = 0
        self.cta_gen = 0

    # TMA: a copy into `buffer` of the tile of `step`
    def copy(self, bar, buffer, step):
        check(self.readers.get(buffer, 0) == 0, "TMA overwrites a buffer an MMA still reads", buffer, step)
        self.buf[buffer] = None
        bar.arrive(tx=1)
        self.tma.append((bar, buffer, step))

    # tensor pipe: MMAs run in issue order; a commit arrives after all before it
    def mma(self, reads, step, on_done=None):
        for b in reads:
            check(self.buf.get(b) == step, "MMA reads a buffer not holding its step", b, step, self.buf.get(b))
            self.readers[b] = self.readers.get(b, 0) + 1
        self.pipe.append(("mma", reads, on_done))

    def commit(self, bar):
        self.pipe.append(("commit", bar))

    def step_async(self):
        options = [k for k, q in (("tma", self.tma), ("pipe", self.pipe)) if q]
        if not options:
            return False
        if self.rng.choice(options) == "tma":
            bar, buffer, step = self.tma.pop(self.rng.randrange(len(self.tma)))
            self.buf[buffer] = step
            bar.complete_tx(1)
        else:
            op = self.pipe.pop(0)
            if op[0] == "commit":
                op[1].arrive()
            else:
                for b in op[1]:
                    self.readers[b] -= 1
                if op[2]:
                    op[2]()
        return True

    # __syncthreads: generator helper, all warps
    def syncthreads(self):
        gen = self.cta_gen
        self.cta_arrived += 1
        if self.cta_arrived == self.n_warps:
            self.cta_arrived, self.cta_gen = 0, self.cta_gen + 1
        while self.cta_gen == gen:
            yield


def run(machine, roles, limit=400000):
    alive = list(roles)
    for _ in range(limit):
        if not alive and not machine.tma and not machine.pipe:
            return
        if alive and (not (machine.tma or machine.pipe) or machine.rng.random() < 0.6):
            r = machine.rng.choice(alive)
            try:
                next(r)
            except StopIteration:
                alive.remove(r)
        else:
            machine.step_async()
    raise ModelError("no progress: deadlock")


RING = 4          # dK/dV kernel at head dim 128: ring slots of 64-row (Q, dO) tile pairs
N_EW = 4          # elementwise warps modelled (the kernel has 16, one arrival each)


def dkdv_model(nsteps, seed, plant=None, ring=RING):
    """The dK/dV kernel (64-row steps): K, V resident; Q, dO and the step's
    statistics streamed through one ring; S and dP double-buffered.  Per step
    dV(st) [reads S_b], S(st+2) [writes S_b], dK(st) [reads dP_b], ring slot
    released, dP(st+2) [writes dP_b]."""
    RING = ring
    m = Machine(seed)
    res_full, done = Bar("res_full"), Bar("done")
    ring_full = [Bar("ring_full%d" % i) for i in range(RING)]
    ring_empty = [Bar("ring_empty%d" % i) for i in range(RING)]
    s_full = [Bar("s_full%d" % b) for b in range(2)]
    dp_full = [Bar("dp_full%d" % b) for b in range(2)]
    p_full = [Bar("p_full%d" % b, count=N_EW) for b in range(2)]
    # TMEM buffers, per column chunk (warp w owns chunk w of each buffer):
    # what the chunk holds ("S"/"P" or "dP"/"dS", step); and per buffer the
    # unfinished products reading it
    tm = {(x, b, w): None for x in ("S", "D") for b in range(2) for w in range(N_EW)}
    tm_readers = {(x, b): 0 for x in ("S", "D") for b in range(2)}
    stats = [{"step": None, "readers": set()} for _ in range(RING)]

    def par(intended):
        """Parity of completion number `intended` (a planted mistake flips it)."""
        p = intended & 1
        return 1 - p if plant == "wrong_parity" else p

    def write_tm(key, step):      # a product overwriting S_b or dP_b completes
        def f():
            check(tm_readers[key] == 0, "S/dP overwritten before the product reading P/dS ran", key, step)
            for w in range(N_EW):
                tm[key + (w,)] = ("S" if key[0] == "S" else "dP", step)
        return f

    def read_tm(key, step):       # an accumulating product reads P/dS of `step`
        want = ("P" if key[0] == "S" else "dS", step)
        for w in range(N_EW):
            check(tm[key + (w,)] == want, "accumulating product before every warp wrote P/dS", key, w, step,
                  tm[key + (w,)])
        tm_readers[key] += 1

        def f():
            tm_readers[key] -= 1
        return f

    def producer():
        m.buf["res"] = None
        res_full.arrive(tx=1)
        m.tma.append((res_full, "res", 0))
        for st in range(nsteps):
            slot = st % RING
            if st >= RING and plant != "early_copy":
                n = st // RING - 1
                while not ring_empty[slot].ready(par(n), n):
                    yield
            check(not stats[slot]["readers"], "statistics rewritten while read", slot, st)
            stats[slot]["step"] = st
            m.copy(ring_full[slot], ("q", slot), st)
            yield

    def mma():
        while not res_full.ready(0, 0):
            yield

        def wait_in(st):
            n = st // RING
            while not ring_full[st % RING].ready(par(n), n):
                yield

        def issue_s(st):
            m.mma([("q", st % RING)], st, write_tm(("S", st & 1), st))
            m.commit(s_full[st & 1])

        def issue_dp(st):
            m.mma([("q", st % RING)], st, write_tm(("D", st & 1), st))
            m.commit(dp_full[st & 1])

        for st in range(min(2, nsteps)):
            yield from wait_in(st)
            issue_s(st)
            issue_dp(st)
        for st in range(nsteps):
            b, slot, nxt, n = st & 1, st % RING, st + 2 < nsteps, st >> 1
            while not p_full[b].ready(par(n), n):
                yield
            if nxt:
                yield from wait_in(st + 2)
            if plant == "early_overwrite" and nxt:
                issue_s(st + 2)
            m.mma([("q", slot)], st, read_tm(("S", b), st))             # dV += P^T dO
            if nxt and plant != "early_overwrite":
                issue_s(st + 2)
            m.mma([("q", slot)], st, read_tm(("D", b), st))             # dK += dS^T Q
            m.commit(ring_empty[slot])
            if nxt:
                issue_dp(st + 2)
            yield
        m.commit(done)

    def elementwise(w):
        for st in range(nsteps):
            b, slot, n, nr = st & 1, st % RING, st >> 1, st // RING
            while not ring_full[slot].ready(par(nr), nr):
                yield
            check(stats[slot]["step"] == st, "statistics of another step", w, st, stats[slot]["step"])
            stats[slot]["readers"].add(w)
            while not s_full[b].ready(par(n), n):
                yield
            check(tm[("S", b, w)] == ("S", st), "elementwise reads S before its product", w, st, tm[("S", b, w)])
            yield
            tm[("S", b, w)] = ("P", st)           # P^T over this warp's chunk of S_b
            while not dp_full[b].ready(par(n), n):
                yield
            check(tm[("D", b, w)] == ("dP", st), "elementwise reads dP before its product", w, st, tm[("D", b, w)])
            yield
            tm[("D", b, w)] = ("dS", st)          # dS^T over its chunk of dP_b
            stats[slot]["readers"].discard(w)
            p_full[b].arrive()
            yield
        if nsteps > 0:
            while not done.ready(0, 0):
                yield

    run(m, [producer(), mma()] + [elementwise(w) for w in range(N_EW)])
    check(not m.pipe and not m.tma, "work left in flight at exit")


RING_K, RING_V = 3, 2   # dQ kernel at head dim 128: K and V rings of 128-row tiles


def dq_model(nsteps, seed, plant=None):
    """The dQ kernel (128-key steps): Q, dO resident; K and V in separate
    rings; S double-buffered, dP single (free once every warp has read it).
    Per step: dP(jt+1) [after the weights of jt], dQ(jt) [reads dS over S_b],
    K's slot released, S(jt+2) [overwrites S_b].  The rows' O tile lands in
    the last V slot first; half of the elementwise warps read it (with the
    resident dO) for D_i, all of them meet at a named barrier, and one arrival
    on o_free lets the producer load that slot's first V tile."""
    m = Machine(seed)
    res_full, done = Bar("res_full"), Bar("done")
    o_full, o_free = Bar("o_full"), Bar("o_free")
    o_slot = ("v", RING_V - 1)
    ew_bar = {"arrived": 0, "gen": 0}
    k_full = [Bar("k_full%d" % i) for i in range(RING_K)]
    k_empty = [Bar("k_empty%d" % i) for i in range(RING_K)]
    v_full = [Bar("v_full%d" % i) for i in range(RING_V)]
    v_empty = [Bar("v_empty%d" % i) for i in range(RING_V)]
    s_full = [Bar("s_full%d" % b) for b in range(2)]
    dp_full = Bar("dp_full")
    p_full = [Bar("p_full%d" % b, count=N_EW) for b in range(2)]
    tm = {("S", b, w): None for b in range(2) for w in range(N_EW)}
    tm.update({("D", w): None for w in range(N_EW)})
    readers = {("S", b): 0 for b in range(2)}

    def par(intended):
        p = intended & 1
        return 1 - p if plant == "wrong_parity" else p

    def write_s(b, jt):
        def f():
            check(readers[("S", b)] == 0, "S overwritten before the dQ product reading dS ran", b, jt)
            for w in range(N_EW):
                tm[("S", b, w)] = ("S", jt)
        return f

    def write_dp(jt):
        def f():
            for w in range(N_EW):
                check(jt == 0 or tm[("D", w)] == ("read", jt - 1), "dP overwritten before a warp read it", w, jt,
                      tm[("D", w)])
                tm[("D", w)] = ("dP", jt)
        return f

    def read_ds(b, jt):
        for w in range(N_EW):
            check(tm[("S", b, w)] == ("dS", jt), "dQ product before every warp wrote dS", b, w, jt,
                  tm[("S", b, w)])
        readers[("S", b)] += 1

        def f():
            readers[("S", b)] -= 1
        return f

    def producer():
        m.buf["res"] = None
        res_full.arrive(tx=1)
        m.tma.append((res_full, "res", 0))
        m.copy(o_full, o_slot, "O")
        for jt in range(nsteps):
            ks, vs = jt % RING_K, jt % RING_V
            if jt >= RING_K and plant != "early_copy":
                n = jt // RING_K - 1
                while not k_empty[ks].ready(par(n), n):
                    yield
            m.copy(k_full[ks], ("k", ks), jt)
            yield
            if jt >= RING_V:
                n = jt // RING_V - 1
                while not v_empty[vs].ready(par(n), n):
                    yield
            elif ("v", vs) == o_slot and plant != "early_v":
                while not o_free.ready(0, 0):
                    yield
            m.copy(v_full[vs], ("v", vs), jt)
            yield

    def mma():
        while not res_full.ready(0, 0):
            yield

        def issue_s(jt):
            ks, n = jt % RING_K, jt // RING_K
            while not k_full[ks].ready(par(n), n):
                yield
            m.mma([("k", ks)], jt, write_s(jt & 1, jt))
            m.commit(s_full[jt & 1])

        def issue_dp(jt):
            vs, n = jt % RING_V, jt // RING_V
            while not v_full[vs].ready(par(n), n):
                yield
            m.mma([("v", vs)], jt, write_dp(jt))
            m.commit(dp_full)
            m.commit(v_empty[vs])

        if nsteps > 0:
            yield from issue_s(0)
            yield from issue_dp(0)
        if nsteps > 1:
            yield from issue_s(1)
        for jt in range(nsteps):
            b, n = jt & 1, jt >> 1
            if plant == "early_dp" and jt + 1 < nsteps:
                yield from issue_dp(jt + 1)
            while not p_full[b].ready(par(n), n):
                yield
            if jt + 1 < nsteps and plant != "early_dp":
                yield from issue_dp(jt + 1)
            if plant == "early_overwrite" and jt + 2 < nsteps:
                yield from issue_s(jt + 2)
            m.mma([("k", jt % RING_K)], jt, read_ds(b, jt))       # dQ += dS K
            m.commit(k_empty[jt % RING_K])
            if jt + 2 < nsteps and plant != "early_overwrite":
                yield from issue_s(jt + 2)
            yield
        m.commit(done)

    def elementwise(w):
        if w < N_EW // 2:   # D_i from dO (resident) and the O tile
            while not (res_full.ready(0, 0) and o_full.ready(0, 0)):
                yield
            check(m.buf.get(o_slot) == "O", "D_i reads O before it landed", w, m.buf.get(o_slot))
            m.readers[o_slot] = m.readers.get(o_slot, 0) + 1
            yield
            check(m.buf.get(o_slot) == "O", "O overwritten while D_i reads it", w, m.buf.get(o_slot))
            m.readers[o_slot] -= 1
        gen = ew_bar["gen"]   # named barrier of the elementwise warps
        ew_bar["arrived"] += 1
        if ew_bar["arrived"] == N_EW:
            ew_bar["arrived"], ew_bar["gen"] = 0, gen + 1
        while ew_bar["gen"] == gen:
            yield
        if w == 0:
            o_free.arrive()
        for jt in range(nsteps):
            b, n = jt & 1, jt >> 1
            while not s_full[b].ready(par(n), n):
                yield
            check(tm[("S", b, w)] == ("S", jt), "elementwise reads S before its product", w, jt, tm[("S", b, w)])
            yield
            while not dp_full.ready(par(jt), jt):
                yield
            check(tm[("D", w)] == ("dP", jt), "elementwise reads dP before its product", w, jt, tm[("D", w)])
            tm[("D", w)] = ("read", jt)
            yield
            tm[("S", b, w)] = ("dS", jt)
            p_full[b].arrive()
            yield
        if nsteps > 0:
            while not done.ready(0, 0):
                yield

    run(m, [producer(), mma()] + [elementwise(w) for w in range(N_EW)])
    check(not m.pipe and not m.tma, "work left in flight at exit")


@pytest.mark.parametrize("ring", [4, 8])
@pytest.mark.parametrize("n", [0, 1, 2, 3, 4, 5, 9, 17])
def test_dkdv_protocol_holds_under_random_interleavings(n, ring):
    for seed in range(30):
        dkdv_model(n, seed, ring=ring)


@pytest.mark.parametrize("n", [0, 1, 2, 3, 4, 5, 9])
def test_dq_protocol_holds_under_random_interleavings(n):
    for seed in range(30):
        dq_model(n, seed)


@pytest.mark.parametrize("plant", ["early_copy", "wrong_parity", "early_overwrite"])
def test_dkdv_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(20):
        try:
            dkdv_model(7, seed, plant=plant)
        except ModelError:
            caught += 1
    assert caught > 0, plant


@pytest.mark.parametrize("plant", ["early_copy", "wrong_parity", "early_overwrite", "early_dp", "early_v"])
def test_dq_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(20):
        try:
            dq_model(7, seed, plant=plant)
        except ModelError:
            caught += 1
    assert caught > 0, plant
