"""Race check of the tcgen05 extend / prefill kernel's pipeline, on the CPU.

The GPU race checker is not available here, so the kernel's barrier schedule is restated
as a model: every role of one CTA (the K producer that also takes units from the queue,
the V producer that also loads Q, the MMA issuer, and the two softmax warps of one row
group, which split the columns and exchange maxima and sums) runs as a generator of
waits, arrivals and asynchronous operations (TMA loads and stores, MMAs with their
commits). A random scheduler interleaves them; asynchronous operations complete later, in
issue order per issuer. The model asserts on every shared buffer that no write lands
before the last reader of the previous contents is done and that every read sees the
contents it expects, and it reports a deadlock when no role and no operation can move.

Barrier semantics follow the mbarrier's phase parity: a wait on parity p passes once the
phase with that parity has completed (a fresh barrier passes parity 1). One thread's
tensor-core operations complete in issue order (a commit arrives once everything that
thread issued before it is done), so some of the kernel's waits are implied by others and
are kept only as a second guard: the softmax's wait for P(g-2) V(g-2) before it writes
P(g) (s_full(g) already implies it), s_empty (S(g+2) is issued after P(g) V(g), which
needs the softmax to be done with S(g)) and o_empty (a unit's first P V needs P from
warps that have read the previous unit's O). The planted mistakes are on the waits that
nothing else implies. The schedule
mirrors extend_tc_kernel in paged_kv_cache_436_b200/csrc/pa_extend_tc.cu; a change of its
barriers has to be made here as well, and the planted mistakes at the end show that the
model notices each kind of race.
"""

import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        assert self.pending > 0, f"over-arrival on {self.name}"
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


class Race(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise Race(msg)


def simulate(units, seed, fresh=False, mutant=None):
    """units: K/V tiles per unit, in the order the queue hands them to this CTA.
    fresh: whole-prompt prefill (tiles from the prompt rows, some stored to the cache)."""
    rng = random.Random(seed)
    p_complete = rng.uniform(0.05, 0.5)         # how eagerly asynchronous operations land
    SPLIT = 2                                   # softmax warps of one row group
    B = {}
    for b in range(2):
        for n, c in (("k_full", 1), ("v_full", 1), ("k_empty", 1), ("pv_done", 1), ("s_full", 1),
                     ("s_empty", SPLIT), ("p_full", SPLIT), ("o_full", 1), ("o_empty", SPLIT)):
            B[f"{n}{b}"] = Bar(f"{n}{b}", c)
    for n, c in (("q_full", 1), ("q_empty", 1), ("grp", SPLIT)):
        B[n] = Bar(n, c)
    for i in range(4):
        B[f"uq_full{i}"] = Bar(f"uq_full{i}", 1)
        B[f"uq_empty{i}"] = Bar(f"uq_empty{i}", 2 + SPLIT)   # V producer, MMA, softmax warps

    # what each shared buffer holds and who still has to read it
    S = {0: None, 1: None}          # tile whose scores are in S buffer b
    S_readers = {0: set(), 1: set()}
    P = {(b, w): None for b in range(2) for w in range(SPLIT)}   # tile whose P slice is in buffer b
    O = {0: None, 1: None}          # unit accumulating in O buffer ob
    O_readers = {0: set(), 1: set()}
    Kb, Vb = {0: None, 1: None}, {0: None, 1: None}
    Vb_stores = {0: 0, 1: 0}        # cache stores still reading the buffer (fresh)
    Kb_stores = {0: 0, 1: 0}
    Q = [None]
    pub = {}                        # (slot, warp) -> value published for the partner
    uq = [None] * 4
    pv_done_tile = {0: -1, 1: -1}
    s_done_tile = {0: -1, 1: -1}
    units_done = []

    n_units = len(units)
    queue = list(range(n_units)) + [-1]

    def next_unit(k, role, taker=False):
        slot, ph = k & 3, (k >> 2) & 1
        if taker:
            yield ("wait", f"uq_empty{slot}", ph ^ 1)
            u = queue[min(k, n_units)]
            uq[slot] = u
            yield ("arrive", f"uq_full{slot}")
            return u
        yield ("wait", f"uq_full{slot}", ph)
        u = uq[slot]
        yield ("arrive", f"uq_empty{slot}")
        return u

    # ---------------- producers ----------------
    def producer(is_v):
        g = 0
        full, empty, buf = ("v_full", "pv_done", Vb) if is_v else ("k_full", "k_empty", Kb)
        stores = Vb_stores if is_v else Kb_stores
        pend = None
        k = 0
        while True:
            u = yield from next_unit(k, "V" if is_v else "K", taker=not is_v)
            if u < 0:
                break
            if is_v:
                if k > 0 and mutant != "q_reload_early":
                    yield ("wait", "q_empty", (k - 1) & 1)

                def q_load(u=u):
                    Q[0] = u
                yield ("async", "q_full", q_load)
            for j in range(units[u]):
                b = g & 1
                if mutant != ("v_reload_early" if is_v else "k_reload_early"):
                    yield ("wait", f"{empty}{b}", ((g >> 1) & 1) ^ 1)
                if fresh:
                    # every store that read the buffers is done before a buffer is reloaded
                    while stores[b] > 0 and mutant != "store_not_waited":
                        yield ("spin",)

                def issue(b=b, g=g):   # the copy starts writing the buffer when it is issued
                    check(stores[b] == 0, f"{'V' if is_v else 'K'} buffer {b} reloaded under a cache store")
                    if is_v:
                        check(pv_done_tile[b] >= g - 2, f"V buffer {b} reloaded before P V of tile {g - 2}")
                    else:
                        check(s_done_tile[b] >= g - 2, f"K buffer {b} reloaded before S of tile {g - 2}")
                    buf[b] = None

                def land(b=b, g=g):
                    buf[b] = g
                yield ("act", issue)
                yield ("async", f"{full}{b}", land)
                if fresh and pend is not None:
                    pb, pg = pend
                    yield ("wait", f"{full}{pb}", (pg >> 1) & 1)
                    stores[pb] += 1

                    def store_done(pb=pb, pg=pg):
                        check(buf[pb] == pg, f"cache store of tile {pg} read a reloaded buffer")
                        stores[pb] -= 1
                    yield ("async", None, store_done)
                    pend = None
                if fresh and j % 2 == 0:        # this unit writes some of its tiles to the cache
                    pend = (b, g)
                g += 1
            k += 1
        if fresh and pend is not None:
            pb, pg = pend
            yield ("wait", f"{full}{pb}", (pg >> 1) & 1)
            stores[pb] += 1

            def store_done(pb=pb, pg=pg):
                stores[pb] -= 1
            yield ("async", None, store_done)

    # ---------------- MMA issuer ----------------
    def mma():
        g, k = 0, 0
        while True:
            u = yield from next_unit(k, "MMA")
            if u < 0:
                break
            ob = k & 1
            yield ("wait", "q_full", k & 1)
            yield ("wait", f"o_empty{ob}", ((k >> 1) & 1) ^ 1)
            n = units[u]

            def pv(h, first, ob=ob, k=k):
                b = h & 1
                yield ("wait", f"p_full{b}", (h >> 1) & 1)
                yield ("wait", f"v_full{b}", (h >> 1) & 1)

                def act(h=h, b=b):
                    check(all(P[(b, w)] == h for w in range(SPLIT)), f"P V of tile {h} reads another P")
                    check(Vb[b] == h, f"P V of tile {h} reads another V tile")
                    if first:
                        check(not O_readers[ob], f"O buffer {ob} restarted while unit {O[ob]} is read")
                        O[ob] = k
                    else:
                        check(O[ob] == k, "P V into another unit's accumulator")
                yield ("act", act)

                def done(h=h, b=b):
                    pv_done_tile[b] = h
                yield ("async", f"pv_done{b}", done)

            for j in range(n):
                b = g & 1
                yield ("wait", f"k_full{b}", (g >> 1) & 1)
                yield ("wait", f"s_empty{b}", ((g >> 1) & 1) ^ 1)

                def s_act(g=g, b=b, u=u):
                    check(not S_readers[b], f"S buffer {b} overwritten while tile {S[b]} is read")
                    check(Kb[b] == g, f"S of tile {g} reads another K tile")
                    check(Q[0] == u, "S reads the Q tile of another unit")

                def s_land(g=g, b=b):
                    S[b] = g
                    S_readers[b] = set(range(SPLIT))
                    s_done_tile[b] = g
                yield ("act", s_act)
                yield ("async", f"s_full{b}", s_land)
                yield ("async", f"k_empty{b}", None)
                if j + 1 == n:
                    yield ("async", "q_empty", None)
                if j > 0:
                    yield from pv(g - 1, j == 1)
                g += 1
            yield from pv(g - 1, n == 1)

            def o_land(ob=ob):
                O_readers[ob] = set(range(SPLIT))
            yield ("async", f"o_full{ob}", o_land)
            k += 1

    # ---------------- softmax warps of one row group ----------------
    def softmax(w):
        g, k, xc = 0, 0, 0
        while True:
            u = yield from next_unit(k, f"SM{w}")
            if u < 0:
                break
            ob = k & 1
            n = units[u]
            for j in range(n):
                b = g & 1
                yield ("wait", f"s_full{b}", (g >> 1) & 1)
                yield ("act", lambda g=g, b=b: check(S[b] == g, f"softmax read S of tile {S[b]}, not {g}"))

                def publish(slot, val):
                    pub[(slot, w)] = val
                yield ("act", lambda b=b, g=g: publish(("S", b), g))
                yield ("arrive", "grp")
                yield ("wait", f"pv_done{b}", ((g >> 1) & 1) ^ 1)

                def p_write(b=b, g=g):
                    prev = P[(b, w)]
                    check(prev is None or pv_done_tile[b] >= prev, f"P buffer {b} rewritten before P V of tile {prev}")
                    P[(b, w)] = g
                yield ("act", p_write)
                if mutant != "grp_not_waited":
                    yield ("wait", "grp", xc & 1)
                xc += 1
                yield ("act", lambda b=b, g=g: check(pub.get((("S", b), 1 - w)) == g,
                                                     f"partner's maximum of tile {g} was overwritten"))
                yield ("act", lambda b=b: S_readers[b].discard(w))
                yield ("arrive", f"s_empty{b}")
                if j > 0 and rng.random() < 0.3:   # the reference maximum moved: rescale O
                    if mutant != "rescale_not_waited":
                        yield ("wait", f"pv_done{(g - 1) & 1}", ((g - 1) >> 1) & 1)
                    yield ("act", lambda g=g: check(pv_done_tile[(g - 1) & 1] >= g - 1, "O rescaled under a P V"))
                if j == n - 1 and rng.random() < 0.5:   # a ragged tile: zero the V rows past the end
                    if mutant != "zero_before_v_lands":
                        yield ("wait", f"v_full{b}", (g >> 1) & 1)
                    yield ("act", lambda b=b, g=g: check(Vb[b] == g, f"zeroed rows of another V tile"))
                yield ("arrive", f"p_full{b}")
                g += 1
            if mutant != "o_read_early":
                yield ("wait", f"o_full{ob}", (k >> 1) & 1)
            yield ("act", lambda ob=ob, k=k: check(O[ob] == k and w in O_readers[ob],
                                                   f"read O of unit {O[ob]}, not {k}"))
            yield ("act", lambda ob=ob, k=k: pub.__setitem__((("O", ob), w), k))
            yield ("arrive", "grp")
            yield ("wait", "grp", xc & 1)
            xc += 1
            yield ("act", lambda ob=ob, k=k: check(pub.get((("O", ob), 1 - w)) == k,
                                                   "partner's sum was overwritten"))
            yield ("act", lambda ob=ob: O_readers[ob].discard(w))
            yield ("arrive", f"o_empty{ob}")
            # the output rows are staged in P buffer 0, this warp's own slice: every P V of
            # the unit has completed (o_full), and the next P(g) of buffer 0 is this warp's
            if w == 0:
                units_done.append(u)
            k += 1

    roles = {"K": producer(False), "V": producer(True), "MMA": mma()}
    for w in range(SPLIT):
        roles[f"SM{w}"] = softmax(w)
    waiting = {r: None for r in roles}
    resume = {r: None for r in roles}
    done = set()
    pending = []                       # (issuer, seq, bar, callback)
    seq = 0
    for step in range(2_000_000):
        ready = [r for r in roles if r not in done and
                 (waiting[r] is None or (waiting[r][0] == "wait" and B[waiting[r][1]].passed(waiting[r][2]))
                  or waiting[r][0] == "spin")]
        if not ready and not pending:
            if len(done) == len(roles):
                break
            raise Race(f"deadlock: {[(r, waiting[r]) for r in roles if r not in done]}")
        if pending and (not ready or rng.random() < p_complete):
            issuer = rng.choice(sorted({p[0] for p in pending}))
            i = min(i for i, p in enumerate(pending) if p[0] == issuer)
            _, _, bar, cb = pending.pop(i)
            if cb is not None:
                cb()
            if bar is not None:
                B[bar].arrive()
            continue
        if not ready:
            continue
        r = rng.choice(ready)
        waiting[r] = None
        try:
            op = roles[r].send(resume[r]) if resume[r] is not None else next(roles[r])
        except StopIteration:
            done.add(r)
            continue
        resume[r] = None
        kind = op[0]
        if kind in ("wait", "spin"):
            waiting[r] = op
        elif kind == "arrive":
            B[op[1]].arrive()
        elif kind == "async":
            seq += 1
            pending.append((r, seq, op[1], op[2]))
        elif kind == "act":
            if op[1] is not None:
                op[1]()
    else:
        raise Race("no progress bound reached")
    check(sorted(units_done) == list(range(n_units)), "not every unit finished")
    check(all(v == 0 for v in Kb_stores.values()) and all(v == 0 for v in Vb_stores.values()),
          "cache stores still in flight at the end")


def _workloads(n, seed):
    rng = random.Random(seed)
    return [[rng.choice([1, 1, 2, 3, 4, 7, 16]) for _ in range(rng.randint(1, 9))] for _ in range(n)]


@pytest.mark.parametrize("fresh", [False, True])
def test_schedule_has_no_race_and_no_deadlock(fresh):
    for i, units in enumerate(_workloads(300, 7 + fresh)):
        simulate(units, seed=i, fresh=fresh)


@pytest.mark.parametrize("mutant,fresh", [
    ("k_reload_early", False),       # K(g+2) loaded before S(g) has read the buffer
    ("v_reload_early", False),       # V(g+2) loaded before P(g) V(g) has read the buffer
    ("q_reload_early", False),       # the next unit's Q loaded before this unit's last S
    ("rescale_not_waited", False),   # O rescaled while P(g-1) V(g-1) may still add to it
    ("zero_before_v_lands", False),  # V rows zeroed before the tile's load has landed
    ("grp_not_waited", False),       # the partner's maximum read before it was published
    ("o_read_early", False),         # O read out before the unit's last P V completed
    ("store_not_waited", True),      # a K/V buffer reloaded while a cache store still reads it
])
def test_planted_schedule_mistakes_are_caught(mutant, fresh):
    with pytest.raises(Race):
        for i, units in enumerate(_workloads(300, 11)):
            simulate(units, seed=i, fresh=fresh, mutant=mutant)
