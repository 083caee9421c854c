"""Model check of the two-tile forward kernel's synchronisation protocol (no GPU).

compute-sanitizer is not available for the kernels, so the protocol of
csrc/sdpa_fwd2q_sm100.cuh (one-warp form) is restated here as a discrete-event
model -- the TMA producer, the single MMA-issuing thread, the two softmax
stages, the epilogue, the TMA engine and the in-order tensor pipe -- and run
under many random interleavings.  The model follows the kernel's roles:

- producer: per unit, each active stage's Q tile into its buffer (after that
  buffer's previous unit's last Q K^T), then the unit's K_j V_j tiles in stream
  order through one ring (a slot reused after the products reading it);
- MMA thread: a prologue Q K^T on the first K tile, then per V tile in stream
  order, per stage, O_s (+)= P_s V (after P_s, and for a unit's first tile after
  the epilogue has read the previous O_s) and S_s = Q_s K^T of the next K tile;
  the step's K/V slot releases are committed at the top of the next step;
- softmax stage s: per tile, S_s is read and P_s written over it (O_s may be
  rescaled in place); per unit the row statistics go to the epilogue;
- epilogue: per unit and stage, the statistics, then O_s once complete.

Checked at every event: a parity wait succeeds only on the completion it
means; a copy never lands in a buffer an issued, unfinished product reads, and
every product reads the tiles of its own unit and tile; S_s is read only when
it holds this tile's scores and is overwritten only after the product reading
P_s ran; P_s is read only after the softmax wrote it; O_s is rescaled only
after the previous product into it ran, restarted only after the epilogue read
it, and read by the epilogue only when complete; the statistics are not
rewritten before they are read; nothing deadlocks and nothing is in flight at
exit.  A second, smaller model covers the split form's exchange of tile
maxima between the two half warps of a row (a two-parity slot and a two-warp
barrier).  Planted mistakes must be caught, so the models are known to be able
to fail.
"""
import random

import pytest

from test_bwd_protocol_model import Bar, Machine, ModelError, check, run

NS = 5      # K/V ring slots (16-bit head dim 128)


def fwd_model(units, seed, qb_count=1, plant=None):
    """units: list of (n0, n1), the K/V tiles of stage 0 and stage 1 of each
    unit (a causal unit has n0 = n1 - 1; a unit whose second query tile lies
    past Sq has n1 = 0); the unit's stream holds max(n0, n1) tiles."""
    m = Machine(seed)
    QB = qb_count
    q_full = [[Bar("q_full%d%d" % (s, b)) for b in range(QB)] for s in range(2)]
    q_empty = [[Bar("q_empty%d%d" % (s, b)) for b in range(QB)] for s in range(2)]
    kv_full = [Bar("kv_full%d" % i) for i in range(NS)]
    kv_empty = [Bar("kv_empty%d" % i) for i in range(NS)]
    s_full = [Bar("s_full%d" % s) for s in range(2)]
    p_full = [Bar("p_full%d" % s) for s in range(2)]
    o_full = [Bar("o_full%d" % s) for s in range(2)]
    o_empty = [Bar("o_empty%d" % s) for s in range(2)]
    st_full = [Bar("st_full%d" % s) for s in range(2)]
    st_empty = [Bar("st_empty%d" % s) for s in range(2)]
    # TMEM per stage: S_s ("S"/"P"/"Pread", unit, tile) and O_s ((unit, last
    # tile accumulated) or "read"); the statistics hand-off per stage
    S = [None, None]
    O = [None, None]
    stats = [None, None]

    def tiles(u, s):
        return units[u][s]

    def n_of(u):
        return max(units[u])

    def par(intended):
        p = intended & 1
        return 1 - p if plant == "wrong_parity" else p

    def wait(bar, n):
        while not bar.ready(par(n), n):
            yield

    def mma(reads, on_issue, on_done):
        """Issue a product reading smem buffers [(buffer, expected content)]."""
        for b, want in reads:
            check(m.buf.get(b) == want, "product reads a buffer not holding its tile", b, want, m.buf.get(b))
            m.readers[b] = m.readers.get(b, 0) + 1
        on_issue()

        def done():
            for b, _ in reads:
                m.readers[b] -= 1
            on_done()
        m.pipe.append(("mma", [], done))

    def stream():
        for u in range(len(units)):
            for j in range(n_of(u)):
                yield u, j

    # ---------------------------------------------------------------- producer
    def producer():
        kq = [0, 0]
        t = 0
        for u in range(len(units)):
            for s in range(2):
                if tiles(u, s) == 0:
                    continue
                qb, use = kq[s] % QB, kq[s] // QB
                if use >= 1:
                    yield from wait(q_empty[s][qb], use - 1)
                m.copy(q_full[s][qb], ("q", s, qb), (u, s))
                kq[s] += 1
                yield
            for j in range(n_of(u)):
                for kind in ("K", "V"):
                    slot = t % NS
                    if t >= NS:
                        yield from wait(kv_empty[slot], t // NS - 1)
                    m.copy(kv_full[slot], ("kv", slot), (u, j, kind))
                    t += 1
                    yield

    # ---------------------------------------------------------------- MMA
    def mma_thread():
        cp = [0, 0]      # P_s consumed
        kqk = [0, 0]     # units started, QK side
        kpv = [0, 0]     # units started, PV side

        def qk_stage(u, j, s, slot):
            qb = kqk[s] % QB
            if j == 0:
                yield from wait(q_full[s][qb], kqk[s] // QB)

            def issue():
                pass

            def done(u=u, j=j, s=s):
                check(S[s] is None or S[s][0] == "Pread", "S overwritten before the product reading P ran",
                      s, u, j, S[s])
                S[s] = ("S", u, j)
            mma([(("q", s, qb), (u, s)), (("kv", slot), (u, j, "K"))], issue, done)
            m.commit(s_full[s])
            last = j == tiles(u, s) - 1
            if (plant == "early_q_empty" and j == 0) or (plant != "early_q_empty" and last):
                m.commit(q_empty[s][qb])
            if last:
                kqk[s] += 1

        def pv_stage(u, j, s, slot):
            yield from wait(p_full[s], cp[s])
            if j == 0 and kpv[s] > 0 and plant != "no_o_empty":
                yield from wait(o_empty[s], kpv[s] - 1)

            def issue(u=u, j=j, s=s):
                check(S[s] == ("P", u, j), "P read before the softmax wrote it", s, u, j, S[s])

            def done(u=u, j=j, s=s):
                S[s] = ("Pread", u, j)
                if j == 0:
                    check(O[s] is None or O[s] == "read", "O restarted before the epilogue read it", s, u, O[s])
                else:
                    check(O[s] == (u, j - 1), "O accumulates out of order", s, u, j, O[s])
                O[s] = (u, j)
            mma([(("kv", slot), (u, j, "V"))], issue, done)
            if j == tiles(u, s) - 1:
                m.commit(o_full[s])
                kpv[s] += 1
            cp[s] += 1

        pos = list(stream())
        t = 0
        ki = 0           # next K tile in stream order
        if pos:
            u, j = pos[0]
            slot = t % NS
            yield from wait(kv_full[slot], t // NS)
            for s in range(2):
                if tiles(u, s) > 0:
                    yield from qk_stage(u, j, s, slot)
            m.commit(kv_empty[slot])
            t += 1
            ki = 1
        pend = []
        for vi in range(len(pos)):
            u, j = pos[vi]
            slot_v = t % NS
            if plant == "early_release":
                m.commit(kv_empty[slot_v])      # the slot freed before its V is read
            yield from wait(kv_full[slot_v], t // NS)
            for b in pend:
                m.commit(kv_empty[b])
            pend = []
            slot_k = (t + 1) % NS
            k_ready = False
            ku, kj = pos[ki] if ki < len(pos) else (None, None)
            for s in range(2):
                if plant == "qk_before_pv" and ku is not None and kj < tiles(ku, s):
                    if not k_ready:
                        yield from wait(kv_full[slot_k], (t + 1) // NS)
                        k_ready = True
                    yield from qk_stage(ku, kj, s, slot_k)
                if j < tiles(u, s):
                    yield from pv_stage(u, j, s, slot_v)
                if plant != "qk_before_pv" and ku is not None and kj < tiles(ku, s):
                    if not k_ready:
                        yield from wait(kv_full[slot_k], (t + 1) // NS)
                        k_ready = True
                    yield from qk_stage(ku, kj, s, slot_k)
            if plant != "early_release":
                pend.append(slot_v)
            t += 1
            if ku is not None:
                pend.append(slot_k)
                t += 1
                ki += 1
            yield
        for b in pend:
            m.commit(kv_empty[b])

    # ---------------------------------------------------------------- softmax
    def softmax(s):
        cs = 0
        ks = 0
        for u in range(len(units)):
            for j in range(tiles(u, s)):
                yield from wait(s_full[s], cs)
                check(S[s] == ("S", u, j), "softmax reads S before its product", s, u, j, S[s])
                if j > 0:   # a rescale of O_s in place needs the previous product done
                    check(O[s] == (u, j - 1), "O rescaled before the previous product ran", s, u, j, O[s])
                yield
                S[s] = ("P", u, j)
                p_full[s].arrive()
                cs += 1
            if tiles(u, s) == 0:
                continue
            if ks > 0:
                yield from wait(st_empty[s], ks - 1)
            check(stats[s] is None or stats[s] == "read", "statistics rewritten before they were read", s, u)
            stats[s] = u
            st_full[s].arrive()
            ks += 1

    # ---------------------------------------------------------------- epilogue
    def epilogue():
        ks = [0, 0]
        for u in range(len(units)):
            for s in range(2):
                if tiles(u, s) == 0:
                    continue
                yield from wait(st_full[s], ks[s])
                check(stats[s] == u, "epilogue reads another unit's statistics", s, u, stats[s])
                stats[s] = "read"
                st_empty[s].arrive()
                yield from wait(o_full[s], ks[s])
                check(O[s] == (u, tiles(u, s) - 1), "epilogue reads O before it is complete", s, u, O[s])
                yield
                O[s] = "read"
                o_empty[s].arrive()
                ks[s] += 1

    run(m, [producer(), mma_thread(), softmax(0), softmax(1), epilogue()])
    check(not m.pipe and not m.tma, "work left in flight at exit")


CASES = {
    "one_tile_units": [(1, 1)] * 4,
    "long_units": [(5, 5), (7, 7)],
    "causal_pairs": [(7, 8), (1, 2), (5, 6), (3, 4)],
    "second_tile_past_sq": [(3, 3), (2, 0), (1, 1), (2, 0)],
    "mixed": [(1, 1), (6, 6), (2, 0), (3, 4), (1, 2), (9, 9)],
}


@pytest.mark.parametrize("qb", [1, 2])
@pytest.mark.parametrize("name", sorted(CASES))
def test_fwd_protocol_holds_under_random_interleavings(name, qb):
    for seed in range(25):
        fwd_model(CASES[name], seed, qb_count=qb)


def test_fwd_protocol_random_unit_sequences():
    rng = random.Random(7)
    for seed in range(40):
        units = []
        for _ in range(rng.randrange(1, 6)):
            kind = rng.randrange(3)
            n = rng.randrange(1, 8)
            units.append((n, n) if kind == 0 else (n, n + 1) if kind == 1 else (n, 0))
        fwd_model(units, seed, qb_count=rng.choice([1, 2]))


@pytest.mark.parametrize("plant", ["wrong_parity", "early_release", "qk_before_pv", "no_o_empty", "early_q_empty"])
def test_fwd_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(30):
        try:
            fwd_model(CASES["mixed"], seed, plant=plant)
        except ModelError:
            caught += 1
    assert caught > 0, plant


def xchg_model(ntiles, seed, plant=None):
    """The split form's tile-max exchange within one stage and lane quarter:
    two half warps (keys 0-63 and 64-127 of the same rows) each write their
    tile max into slot (tile parity, half), arrive on a shared barrier
    (count 2) and, once both have, read the other half's value.  The slot of
    a tile parity is rewritten two tiles later, which the barrier of the tile
    in between orders after the other half's read."""
    m = Machine(seed)
    xbar = Bar("xchg", count=2)
    slots = {}

    def par(intended):
        p = intended & 1
        return 1 - p if plant == "wrong_parity" else p

    def half(h):
        for cs in range(ntiles):
            slot = (0 if plant == "single_buffer" else cs & 1, h)
            slots[slot] = (h, cs)
            yield
            xbar.arrive()
            while not xbar.ready(par(cs), cs):
                yield
            other = (slot[0], 1 - h)
            yield
            check(slots.get(other) == (1 - h, cs), "exchange slot holds another tile's max", h, cs, slots.get(other))
            yield

    run(m, [half(0), half(1)])


@pytest.mark.parametrize("n", [1, 2, 3, 8, 17])
def test_xchg_protocol_holds(n):
    for seed in range(40):
        xchg_model(n, seed)


@pytest.mark.parametrize("plant", ["single_buffer", "wrong_parity"])
def test_xchg_planted_mistakes_are_caught(plant):
    caught = 0
    for seed in range(40):
        try:
            xchg_model(8, seed, plant=plant)
        except ModelError:
            caught += 1
    assert caught > 0, plant
