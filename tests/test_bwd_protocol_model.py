"""Model check of the backward kernels' synchronisation protocol (no GPU).

compute-sanitizer is not available for these kernels, so the protocol they
follow -- mbarrier phases, the double-buffered streamed tiles, the queued MMA
commits and the CTA barriers -- is restated here as a small discrete-event
model and run under many random interleavings of the warps, the TMA engine
and the in-order tensor pipe.  The model checks, at every step:

- a parity wait only succeeds on the phase it means (never one phase early,
  never aliased two phases late);
- a TMA copy never lands in a buffer an issued, unfinished MMA still reads,
  and every MMA reads the tile of its own step;
- the elementwise warps read S/dP only after the MMAs that produce them
  completed, and the accumulating MMAs read P/dS only after every warp wrote
  them;
- the per-step statistics are not overwritten while a warp still reads them;
- every role finishes (no deadlock).

Planted mistakes (a copy issued before its buffer is free, a wrong parity)
must be caught, so the model is known to be able to fail.  Each role mirrors
the kernel it is named after in csrc/sdpa_bwd_tc_sm100.cuh.
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


# ---------------------------------------------------------------------------
# dK/dV kernel: K, V once; Q/dO tiles of step s in buffer s & 1; one commit
# per step queues dV/dK of step s and S^T/dP^T of step s+1; LSE/D of the
# step's rows in one shared buffer, rewritten by warps 1-7 after the barrier
# that ends the step's reads.
# ---------------------------------------------------------------------------
def dkdv_model(nsteps, seed, plant=None):
    m = Machine(seed)
    bar_kv, bar_mma = Bar("kv"), Bar("mma")
    bar_in = [Bar("in0"), Bar("in1")]
    tm = {"S": None, "P": None, "P_writers": set()}     # TMEM S^T/dP^T and P^T/dS^T
    stats = {"step": None, "readers": set()}

    def mma1_done(s):
        def f():
            tm["S"] = s
        return f

    def issue_qk(s):           # warp 0: wait for step s's tiles, queue S^T, dP^T
        b = s & 1
        par = (s >> 1) & 1 if plant != "wrong_parity" else 1 - ((s >> 1) & 1)
        while not bar_in[b].ready(par, s >> 1):
            yield
        m.mma([("q", b)], s, mma1_done(s))

    def warp(w):
        if w == 0:
            bar_kv.arrive(tx=1)
            m.tma.append((bar_kv, "kv", 0))
            if nsteps > 0:
                m.copy(bar_in[0], ("q", 0), 0)
        while not bar_kv.ready(0, 0):
            yield
        yield from m.syncthreads()
        if nsteps > 0:
            if w != 0:
                stats["step"] = 0
            if w == 0:
                yield from issue_qk(0)
                m.commit(bar_mma)
        for it in range(nsteps):
            if plant == "early_copy" and w == 0 and it + 1 < nsteps:
                m.copy(bar_in[(it + 1) & 1], ("q", (it + 1) & 1), it + 1)
            while not bar_mma.ready(it & 1, it):
                yield
            yield from m.syncthreads()
            if w == 0 and it + 1 < nsteps and plant != "early_copy":
                m.copy(bar_in[(it + 1) & 1], ("q", (it + 1) & 1), it + 1)
            # elementwise: S^T/dP^T of step it, statistics of step it
            check(tm["S"] == it, "elementwise reads S before its MMAs", w, it, tm["S"])
            check(stats["step"] == it, "statistics of another step", w, it, stats["step"])
            stats["readers"].add(w)
            yield
            stats["readers"].discard(w)
            if tm["P"] != it:
                tm["P"], tm["P_writers"] = it, set()
            tm["P_writers"].add(w)
            yield from m.syncthreads()
            if w == 0:
                check(tm["P_writers"] == set(range(8)), "dV/dK MMAs before every warp wrote P", it)
                m.mma([("q", it & 1)], it)
                if it + 1 < nsteps:
                    yield from issue_qk(it + 1)
                m.commit(bar_mma)
            if it + 1 < nsteps and w != 0:
                check(not stats["readers"], "statistics rewritten while read", w, it)
                stats["step"] = it + 1
        if nsteps > 0:
            while not bar_mma.ready(nsteps & 1, nsteps):
                yield
        yield from m.syncthreads()

    run(m, [warp(w) for w in range(8)])
    check(not m.pipe and not m.tma, "work left in flight at exit")


# ---------------------------------------------------------------------------
# dQ kernel: Q, dO once; K/V tiles of tile j in buffer j & 1; one commit per
# tile queues dQ of tile j and S/dP of tile j+1.
# ---------------------------------------------------------------------------
def dq_model(ntiles, seed, plant=None):
    m = Machine(seed)
    bar_in, bar_mma = Bar("in"), Bar("mma")
    bar_kv = [Bar("kv0"), Bar("kv1")]
    tm = {"S": None, "P_writers": set(), "P": None}

    def mma1_done(j):
        def f():
            tm["S"] = j
        return f

    def issue_qk(j):
        b = j & 1
        par = (j >> 1) & 1 if plant != "wrong_parity" else 1 - ((j >> 1) & 1)
        while not bar_kv[b].ready(par, j >> 1):
            yield
        m.mma([("kv", b)], j, mma1_done(j))

    def warp(w):
        if w == 0:
            bar_in.arrive(tx=1)
            m.tma.append((bar_in, "q", 0))
            if ntiles > 0:
                m.copy(bar_kv[0], ("kv", 0), 0)
        while not bar_in.ready(0, 0):
            yield
        yield from m.syncthreads()
        if ntiles > 0 and w == 0:
            yield from issue_qk(0)
            m.commit(bar_mma)
        for jt in range(ntiles):
            if plant == "early_copy" and w == 0 and jt + 1 < ntiles:
                m.copy(bar_kv[(jt + 1) & 1], ("kv", (jt + 1) & 1), jt + 1)
            while not bar_mma.ready(jt & 1, jt):
                yield
            yield from m.syncthreads()
            if w == 0 and jt + 1 < ntiles and plant != "early_copy":
                m.copy(bar_kv[(jt + 1) & 1], ("kv", (jt + 1) & 1), jt + 1)
            check(tm["S"] == jt, "elementwise reads S before its MMAs", w, jt, tm["S"])
            yield
            if tm["P"] != jt:
                tm["P"], tm["P_writers"] = jt, set()
            tm["P_writers"].add(w)
            yield from m.syncthreads()
            if w == 0:
                check(tm["P_writers"] == set(range(8)), "dQ MMAs before every warp wrote dS", jt)
                m.mma([("kv", jt & 1)], jt)
                if jt + 1 < ntiles:
                    yield from issue_qk(jt + 1)
                m.commit(bar_mma)
        if ntiles > 0:
            while not bar_mma.ready(ntiles & 1, ntiles):
                yield
        yield from m.syncthreads()

    run(m, [warp(w) for w in range(8)])
    check(not m.pipe and not m.tma, "work left in flight at exit")


@pytest.mark.parametrize("model", [dkdv_model, dq_model], ids=["dkdv", "dq"])
@pytest.mark.parametrize("n", [0, 1, 2, 3, 4, 7])
def test_protocol_holds_under_random_interleavings(model, n):
    for seed in range(30):
        model(n, seed)


@pytest.mark.parametrize("model", [dkdv_model, dq_model], ids=["dkdv", "dq"])
@pytest.mark.parametrize("plant", ["early_copy", "wrong_parity"])
def test_planted_mistakes_are_caught(model, plant):
    caught = 0
    for seed in range(20):
        try:
            model(5, seed, plant=plant)
        except ModelError:
            caught += 1
    assert caught > 0, plant
