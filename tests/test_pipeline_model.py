"""Race check of the tcgen05 extend / prefill kernel's pipeline, on the CPU.

The GPU race checker is not available here, so the kernel's barrier schedule is restated
as a model: every role of one CTA runs as a generator of waits, arrivals and
asynchronous operations (TMA loads and stores, MMAs with their commits):

* a K producer that takes the units from the queue, publishes them in a ring, loads each
  unit's Q and streams K tiles through two buffers (tile g in buffer g % 2); a V producer
  that follows the ring and streams V tiles the same way (for whole prompts each also
  stores some of its tiles to the cache);
* softmax warps in pairs: the two warps of a pair own the same rows, one the first 64
  columns of each tile, the other the last 64. Each reads its half of S(g) from one of
  three S buffers in TMEM (tile g in buffer g % 3), exchanges its row maxima with its
  partner (a slot per exchange, two in rotation, and a two-warp barrier), rescales its
  half of O when the reference maximum moves, flags whether its rows need the tile's
  remainder product, writes its half of P(g) over S(g), zeroes ragged V rows (first
  halves); a unit's O is read out (after the row sums are exchanged) once the first tile
  of the next unit is done, so that the unit's last P V runs meanwhile;
* one MMA issuer (one thread) that polls the barriers without blocking and issues whatever
  is ready:
  S(g) once K(g) has landed and P(g - 3) V(g - 3), which read the S buffer, completed --
  so S runs up to three tiles ahead of the softmax -- and P V(g) once P(g) is written and
  V(g) has landed.

A random scheduler interleaves the roles; asynchronous operations complete later, in
issue order per issuer (a commit arrives once everything its thread issued before it is
done). The model asserts on every shared buffer -- the K and V buffers, the Q buffer, the
three S buffers (which hold P after the softmax), the O accumulator, the exchange slots
-- that no write lands before the last reader of the previous contents is done and that
every read sees the contents it expects; it reports a deadlock when no role and no
operation can move.

Barriers follow the mbarrier's phase parity: a wait names the phase it needs (the kernel
passes that phase's parity) and passes once the phase has completed -- a fresh barrier
passes the wait for phase -1. A parity wait is only sound while the barrier is at most
one phase past the awaited one and not behind it, so the model also fails a wait (or a
non-blocking test) that the parity would let through at any other phase. One of the
kernel's waits is implied by another and kept only as a second guard: a unit's first
P V waits for o_empty, but it also waits for p_full, and the softmax warps write the new
unit's first P only after they have read the previous unit's O. The planted mistakes are
on the waits that nothing else implies. The schedule mirrors extend_tc_kernel in
paged_kv_cache_436_b200/csrc/pa_extend_tc.cu; a change of its barriers has to be made
here as well, and the planted mistakes at the end show that the model notices each kind
of race.
"""

import random

import pytest

NS = 3          # S buffers
NKV = 2         # K and V buffers


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0   # phase: completed phases

    def arrive(self):
        assert self.pending > 0, f"over-arrival on {self.name}"
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def parity_passes(self, n):
        """What the kernel's parity wait for phase n answers."""
        return (self.phase & 1) != (n & 1)


class Race(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise Race(msg)


def simulate(units, seed, fresh=False, mutant=None, quarters=1):
    """units: K/V tiles per unit, in the order the queue hands them out.
    fresh: whole-prompt prefill (tiles from the prompt rows, some stored to the cache).
    quarters: row groups; each has a pair of softmax warps (the kernel has 4 pairs)."""
    rng = random.Random(seed)
    p_complete = rng.uniform(0.05, 0.5)         # how eagerly asynchronous operations land
    W = 2 * quarters                            # softmax warps: warp w pairs with warp (w + quarters) % W
    B = {}
    for b in range(NS):
        for n, cnt in (("s_full", 1), ("p_full", W), ("pv_done", 1)):
            B[f"{n}.{b}"] = Bar(f"{n}.{b}", cnt)
    for x in range(NKV):
        for n in ("k_full", "v_full"):
            B[f"{n}.{x}"] = Bar(f"{n}.{x}", 1)
    for n, cnt in (("q_full", 1), ("q_empty", 1), ("o_full", 1), ("o_empty", W)):
        B[n] = Bar(n, cnt)
    for q in range(quarters):
        B[f"xchg.{q}"] = Bar(f"xchg.{q}", 2)
    for i in range(4):
        B[f"uq_full_{i}"] = Bar(f"uq_full_{i}", 1)
        B[f"uq_empty_{i}"] = Bar(f"uq_empty_{i}", W + 2)   # softmax warps, the MMA warp, the V producer

    def partner(w):
        return w + quarters if w < quarters else w - quarters

    # what each shared buffer holds and how far its readers got
    Kb = [None] * NKV                   # tile in each K buffer
    Vb = [None] * NKV
    Qb = [None]                         # unit whose q rows are in the Q buffer
    S = [None] * NS                     # ("S", g) or ("P", g)
    P_writers = [set() for _ in range(NS)]
    O = [None]                          # unit accumulating in O
    O_readers = set()
    s_done = [-1]                       # last S(g) completed (they complete in order)
    pv_done_t = [-1]                    # last P(g) V(g) completed
    stores = {"K": 0, "V": 0}           # cache stores still reading the K / V buffers
    uq = [None] * 4
    lo_flag = [[(-1, False)] * W for _ in range(NS)]     # (tile, need) per buffer and warp
    xslot = [[None] * W for _ in range(2)]               # exchange slots: the exchange number written
    units_done = []
    queue = {"next": 0}
    n_units = len(units)
    last_s_of_unit = {}

    def owns(j):                        # whole prompts: this unit stores some of its tiles
        return fresh and j % 2 == 0

    # ---------------- K producer: units, Q, K tiles ----------------
    def k_producer():
        g, k = 0, 0
        while True:
            slot = k & 3
            yield ("wait", f"uq_empty_{slot}", (k >> 2) - 1)
            u = queue["next"] if queue["next"] < n_units else -1
            queue["next"] += 1
            uq[slot] = u
            yield ("arrive", f"uq_full_{slot}")
            if u < 0:
                break
            if mutant != "q_reload_early":
                yield ("wait", "q_empty", k - 1)

            def q_issue():
                check(Qb[0] is None or s_done[0] >= last_s_of_unit.get(Qb[0], -1),
                      f"Q buffer reloaded before the last S of unit {Qb[0]}")
                Qb[0] = None

            def q_land(u=u):
                Qb[0] = u
            yield ("act", q_issue)
            yield ("async", "q_full", q_land)
            for j in range(units[u]):
                x = g % NKV
                # K(g) once S(g - 2) has read the buffer
                if g >= NKV and mutant != "k_reload_early":
                    yield ("wait", f"s_full.{(g - NKV) % NS}", (g - NKV) // NS)
                while fresh and stores["K"] > 0 and mutant != "store_not_waited":
                    yield ("spin",)

                def k_issue(g=g, x=x):
                    check(stores["K"] == 0, "K buffer reloaded under a cache store")
                    check(s_done[0] >= g - NKV, f"K buffer {x} reloaded before S of tile {g - NKV}")
                    Kb[x] = None

                def k_land(g=g, x=x):
                    Kb[x] = g
                yield ("act", k_issue)
                yield ("async", f"k_full.{x}", k_land)
                if owns(j):
                    yield ("wait", f"k_full.{x}", g // NKV)
                    stores["K"] += 1

                    def store_done(g=g, x=x):
                        check(Kb[x] == g, f"cache store of K tile {g} read a reloaded buffer")
                        stores["K"] -= 1
                    yield ("async", None, store_done)
                g += 1
            k += 1

    # ---------------- V producer: follows the ring ----------------
    def v_producer():
        g, k = 0, 0
        while True:
            slot = k & 3
            yield ("wait", f"uq_full_{slot}", k >> 2)
            u = uq[slot]
            yield ("arrive", f"uq_empty_{slot}")
            if u < 0:
                break
            for j in range(units[u]):
                x = g % NKV
                # V(g) once P(g - 2) V(g - 2) has read the buffer
                if g >= NKV and mutant != "v_reload_early":
                    yield ("wait", f"pv_done.{(g - NKV) % NS}", (g - NKV) // NS)
                while fresh and stores["V"] > 0 and mutant != "store_not_waited":
                    yield ("spin",)

                def v_issue(g=g, x=x):
                    check(stores["V"] == 0, "V buffer reloaded under a cache store")
                    check(pv_done_t[0] >= g - NKV, f"V buffer {x} reloaded before P V of tile {g - NKV}")
                    Vb[x] = None

                def v_land(g=g, x=x):
                    Vb[x] = g
                yield ("act", v_issue)
                yield ("async", f"v_full.{x}", v_land)
                if owns(j):
                    yield ("wait", f"v_full.{x}", g // NKV)
                    stores["V"] += 1

                    def store_done(g=g, x=x):
                        check(Vb[x] == g, f"cache store of V tile {g} read a reloaded buffer")
                        stores["V"] -= 1
                    yield ("async", None, store_done)
                g += 1
            k += 1

    # ---------------- MMA issuer ----------------
    def mma():
        z = {"s_live": True, "s_fresh": True, "s_j": 0, "s_g": 0, "s_k": 0, "s_u": None,
             "p_fresh": True, "p_j": 0, "p_g": 0, "p_k": 0, "p_u": None}
        released = set()                # units whose ring slot this warp has released

        def try_s():
            if not z["s_live"] or z["s_g"] >= z["p_g"] + NS:
                return False
            if z["s_fresh"]:
                slot = z["s_k"] & 3
                if not (yield ("test", f"uq_full_{slot}", z["s_k"] >> 2)):
                    return False
                u = uq[slot]
                if mutant == "ring_released_early":   # released when the S cursor reads it
                    released.add(z["s_k"])
                    yield ("arrive", f"uq_empty_{slot}")
                if u < 0:
                    z["s_live"] = False
                    return True
                z["s_u"], z["s_j"], z["s_fresh"] = u, 0, False
            g, u = z["s_g"], z["s_u"]
            b, x = g % NS, g % NKV
            if z["s_j"] == 0 and not (yield ("test", "q_full", z["s_k"])):
                return False
            if not (yield ("test", f"k_full.{x}", g // NKV)):
                return False
            if g >= NS and mutant != "s_before_pv_done" and not (yield ("test", f"pv_done.{b}", g // NS - 1)):
                return False

            def s_act(g=g, u=u, b=b, x=x):
                check(Kb[x] == g, f"S of tile {g} reads another K tile")
                check(Qb[0] == u, f"S of unit {u} reads the Q tile of unit {Qb[0]}")
                check(pv_done_t[0] >= g - NS, f"S({g}) overwrites P({g - NS}) while P V reads it")

            def s_land(g=g, b=b):
                S[b] = ("S", g)
                P_writers[b] = set()
                s_done[0] = g
            yield ("act", s_act)
            yield ("async", f"s_full.{b}", s_land)
            if z["s_j"] + 1 == units[u]:
                last_s_of_unit[u] = g
                yield ("async", "q_empty", None)
                z["s_fresh"] = True
                z["s_k"] += 1
            z["s_j"] += 1
            z["s_g"] += 1
            return True

        def try_pv():
            if z["p_g"] >= z["s_g"]:
                return False
            if z["p_fresh"]:
                check(z["p_k"] not in released, f"the P V cursor reads ring slot of unit {z['p_k']} after releasing it")
                z["p_u"], z["p_j"], z["p_fresh"] = uq[z["p_k"] & 3], 0, False
            g, u, j = z["p_g"], z["p_u"], z["p_j"]
            b, x = g % NS, g % NKV
            if mutant != "pv_before_p" and not (yield ("test", f"p_full.{b}", g // NS)):
                return False
            if not (yield ("test", f"v_full.{x}", g // NKV)):
                return False
            if j == 0 and z["p_k"] > 0 and mutant != "o_overwrite_early" and \
                    not (yield ("test", "o_empty", z["p_k"] - 1)):
                return False

            def pv_act(g=g, u=u, j=j, b=b, x=x):
                check(S[b] == ("P", g) and len(P_writers[b]) == W, f"P V of tile {g} reads an unfinished P")
                check(all(t == g for t, _ in lo_flag[b]), f"remainder flags of tile {g} read as {lo_flag[b]}")
                check(Vb[x] == g, f"P V of tile {g} reads another V tile")
                if j == 0:
                    check(not O_readers, f"O restarted while unit {O[0]} is read")
                    O[0] = u
                else:
                    check(O[0] == u, "P V into another unit's accumulator")

            def pv_land(g=g):
                check(pv_done_t[0] == g - 1, "P V products completed out of order")
                pv_done_t[0] = g
            yield ("act", pv_act)
            yield ("async", f"pv_done.{b}", pv_land)
            z["p_g"] += 1
            z["p_j"] += 1
            if z["p_j"] == units[u]:

                def o_land():
                    O_readers.update(range(W))
                yield ("async", "o_full", o_land)
                if mutant != "ring_released_early":
                    released.add(z["p_k"])
                    yield ("arrive", f"uq_empty_{z['p_k'] & 3}")
                z["p_fresh"] = True
                z["p_k"] += 1
            return True

        while z["s_live"] or z["p_g"] < z["s_g"]:
            moved = yield from try_pv()
            moved |= yield from try_s()
            if not moved:
                yield ("spin",)

    # ---------------- softmax warp w: row group w % quarters, column half w // quarters ----------------
    def softmax(w):
        q, h = w % quarters, w // quarters
        g, k, xn = 0, 0, 0

        def exchange():
            nonlocal xn
            s = xn & 1 if mutant != "xchg_one_slot" else 0
            n = xn
            yield ("act", lambda s=s, n=n: xslot[s].__setitem__(w, n))
            yield ("arrive", f"xchg.{q}")
            if mutant != "xchg_not_waited":
                yield ("wait", f"xchg.{q}", n)
            yield ("act", lambda s=s, n=n: check(xslot[s][partner(w)] == n,
                                                 f"warp {w} read exchange {xslot[s][partner(w)]}, not {n}"))
            xn += 1

        def epilogue(kk, uu, gl):
            """Unit kk's O: the row sums exchanged, O read once the unit's last P V completed."""
            if mutant != "o_read_early":
                yield ("wait", "o_full", kk)
            yield from exchange()              # row sums of the two halves
            yield ("act", lambda: check(O[0] == uu and w in O_readers and pv_done_t[0] >= gl,
                                        f"read O of unit {O[0]} before unit {uu} was complete"))
            yield ("act", lambda: O_readers.discard(w))
            yield ("arrive", "o_empty")
            if w == 0:
                units_done.append(uu)

        pend = None                            # the previous unit, whose O is read after this unit's first tile
        while True:
            slot = k & 3
            yield ("wait", f"uq_full_{slot}", k >> 2)
            u = uq[slot]
            yield ("arrive", f"uq_empty_{slot}")
            if u < 0:
                break
            n_t = units[u]
            for j in range(n_t):
                b = g % NS
                yield ("wait", f"s_full.{b}", g // NS)
                yield ("act", lambda g=g, b=b: check(S[b] in (("S", g), ("P", g)), f"softmax read {S[b]}, not S({g})"))
                yield from exchange()          # row maxima of the two halves
                if j > 0 and rng.random() < 0.3:   # the reference maximum moved: rescale O
                    if mutant != "rescale_before_pv_done":
                        yield ("wait", f"pv_done.{(g - 1) % NS}", (g - 1) // NS)
                    yield ("act", lambda g=g: check(pv_done_t[0] >= g - 1, "O rescaled under a P V"))
                need = rng.random() < 0.3

                def flag(g=g, b=b, need=need):
                    lo_flag[b][w] = (g, need)
                if mutant != "flag_after_p_full":
                    yield ("act", flag)

                def p_write(g=g, b=b):
                    check(pv_done_t[0] >= g - NS, f"P({g}) written over P({g - NS}) while P V reads it")
                    S[b] = ("P", g)
                    P_writers[b].add(w)
                yield ("act", p_write)
                if h == 0 and j == n_t - 1 and rng.random() < 0.5:   # a ragged tile: zero the V rows past the end
                    if mutant != "zero_before_v_lands":
                        yield ("wait", f"v_full.{g % NKV}", g // NKV)
                    yield ("act", lambda g=g: check(Vb[g % NKV] == g, "zeroed rows of another V tile"))
                yield ("arrive", f"p_full.{b}")
                if mutant == "flag_after_p_full":
                    yield ("act", flag)
                g += 1
                if j == 0 and pend is not None:
                    yield from epilogue(*pend)
                    pend = None
            pend = (k, u, g - 1)
            k += 1
        if pend is not None:
            yield from epilogue(*pend)

    roles = {"MMA": mma(), "KP": k_producer(), "VP": v_producer()}
    for w in range(W):
        roles[f"SM{w}"] = softmax(w)
    waiting = {r: None for r in roles}
    resume = {r: None for r in roles}
    done = set()
    pending = []                       # (issuer, seq, bar, callback)
    seq = 0

    def parity_state(r, name, n):
        """The kernel's parity answer for phase n of barrier `name`, checked for soundness."""
        bar = B[name]
        if not bar.parity_passes(n):
            check(bar.phase <= n + 1, f"{r} waits for phase {n} of {name}, already at {bar.phase}")
            return False
        check(bar.phase == n + 1, f"{r}: the parity of phase {n} of {name} passes at phase {bar.phase}")
        return True

    def can_go(r):
        op = waiting[r]
        if op is None or op[0] == "spin":
            return True
        return parity_state(r, op[1], op[2])

    for step in range(6_000_000):
        ready = [r for r in roles if r not in done and can_go(r)]
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
        if kind == "test":                # non-blocking: the role continues with the answer
            resume[r] = parity_state(r, op[1], op[2])
        elif kind in ("wait", "spin"):
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
    check(stores["K"] == 0 and stores["V"] == 0, "cache stores still in flight at the end")


def _workloads(n, seed):
    rng = random.Random(seed)
    return [[rng.choice([1, 1, 2, 3, 4, 7, 16]) for _ in range(rng.randint(1, 9))] for _ in range(n)]


@pytest.mark.parametrize("fresh", [False, True])
def test_schedule_has_no_race_and_no_deadlock(fresh):
    for i, units in enumerate(_workloads(300, 7 + fresh)):
        simulate(units, seed=i, fresh=fresh)


def test_schedule_with_four_warp_pairs():
    for i, units in enumerate(_workloads(60, 21)):
        simulate(units, seed=i, fresh=i % 2 == 1, quarters=4)


@pytest.mark.parametrize("mutant,fresh", [
    ("k_reload_early", False),       # K(g) loaded before S(g-2) has read the buffer
    ("v_reload_early", False),       # V(g) loaded before P(g-2) V(g-2) has read the buffer
    ("q_reload_early", False),       # the next unit's Q loaded before this unit's last S
    ("s_before_pv_done", False),     # S(g) written over P(g-3) while P(g-3) V(g-3) reads it
    ("pv_before_p", False),          # P V issued before every warp has written P
    ("o_read_early", False),         # O read out before the unit's last P V completed
    ("zero_before_v_lands", False),  # V rows zeroed before the tile's load has landed
    ("rescale_before_pv_done", False),  # O rescaled while the previous tile's P V may run
    ("flag_after_p_full", False),    # a warp's remainder flag written after it signalled P
    ("xchg_not_waited", False),      # the partner's maxima read before it wrote them
    ("xchg_one_slot", False),        # one exchange slot: overwritten before the partner read it
    ("ring_released_early", False),  # the MMA warp frees a ring slot before its P V cursor read it
    ("store_not_waited", True),      # a K/V buffer reloaded while a cache store still reads it
])
def test_planted_schedule_mistakes_are_caught(mutant, fresh):
    with pytest.raises(Race):
        for i, units in enumerate(_workloads(300, 11)):
            simulate(units, seed=i, fresh=fresh, mutant=mutant)
