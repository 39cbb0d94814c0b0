"""Race check of the tcgen05 extend / prefill kernel's pipeline, on the CPU.

The GPU race checker is not available here, so the kernel's barrier schedule is restated
as a model: every role of one CTA runs as a generator of waits, arrivals and
asynchronous operations (TMA loads and stores, MMAs with their commits):

* per set c (two sets share the tensor core, each working on its own units): a producer
  that takes the set's units from the queue, loads their Q and streams K and V tiles
  through single buffers (and, for whole prompts, stores some tiles to the cache); the
  set's softmax warps, which read S(g) from TMEM, agree whether the tile needs P's
  remainder (a word per tile, three in rotation, and a barrier), write P(g) over S, zero
  ragged V rows, rescale O, and read O out at the end of each unit;
* one MMA issuer for both sets: S of each set's first tile, then in turn for each set
  P V(g) and, once that product has completed, S(g + 1).

A random scheduler interleaves the roles; asynchronous operations complete later, in
issue order per issuer (a commit arrives once everything its thread issued before it is
done). The model asserts on every shared buffer -- the K, V and Q tiles, each set's S
columns (which hold P after the softmax), each set's O accumulator -- that no write lands
before the last reader of the previous contents is done and that every read sees the
contents it expects; it reports a deadlock when no role and no operation can move.

Barrier semantics follow the mbarrier's phase parity: a wait on parity p passes once the
phase with that parity has completed (a fresh barrier passes parity 1). One of the
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

SETS = 2


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


def simulate(units, seed, fresh=False, mutant=None, warps=2):
    """units: K/V tiles per unit, in the order the queue hands them out.
    fresh: whole-prompt prefill (tiles from the prompt rows, some stored to the cache).
    warps: softmax warps per set (the kernel has 4; each arrives once per barrier phase)."""
    rng = random.Random(seed)
    p_complete = rng.uniform(0.05, 0.5)         # how eagerly asynchronous operations land
    B = {}
    for c in range(SETS):
        for n, cnt in (("s_full", 1), ("p_full", warps), ("pv_done", 1), ("k_full", 1), ("v_full", 1),
                       ("k_empty", 1), ("q_full", 1), ("q_empty", 1), ("o_full", 1), ("o_empty", warps),
                       ("vote", warps)):
            B[f"{n}{c}"] = Bar(f"{n}{c}", cnt)
        for i in range(4):
            B[f"uq_full{c}_{i}"] = Bar(f"uq_full{c}_{i}", 1)
            B[f"uq_empty{c}_{i}"] = Bar(f"uq_empty{c}_{i}", warps + 1)   # softmax warps and the MMA warp

    # what each shared buffer holds and how far its readers got
    Kb = [None] * SETS                # tile in the K buffer
    Vb = [None] * SETS
    Qb = [None] * SETS                # unit whose q rows are in the Q buffer
    S = [None] * SETS                 # ("S", g) or ("P", g): the set's S columns
    P_writers = [set() for _ in range(SETS)]
    O = [None] * SETS                 # unit accumulating in the set's O
    O_readers = [set() for _ in range(SETS)]
    s_done = [-1] * SETS              # last S(g) completed
    pv_done_t = [-1] * SETS           # last P(g) V(g) completed
    pv_issued = [-1] * SETS
    stores = [0] * SETS               # cache stores still reading the set's K / V buffers
    uq = [[None] * 4 for _ in range(SETS)]
    vote_word = [[0, 0, 0] for _ in range(SETS)]   # the remainder vote, three words in rotation
    vote_need = [{} for _ in range(SETS)]          # tile -> OR of the warps' needs
    vote_seen = [{} for _ in range(SETS)]          # tile -> the answers the warps read
    units_done = []
    queue = {"next": 0}
    n_units = len(units)

    def next_unit(c, k, taker=False):
        slot, ph = k & 3, (k >> 2) & 1
        if taker:
            yield ("wait", f"uq_empty{c}_{slot}", ph ^ 1)
            u = queue["next"] if queue["next"] < n_units else -1
            queue["next"] += 1
            uq[c][slot] = u
            yield ("arrive", f"uq_full{c}_{slot}")
            return u
        yield ("wait", f"uq_full{c}_{slot}", ph)
        u = uq[c][slot]
        yield ("arrive", f"uq_empty{c}_{slot}")
        return u

    # ---------------- producer of set c ----------------
    def producer(c):
        g = 0
        k = 0
        while True:
            u = yield from next_unit(c, k, taker=True)
            if u < 0:
                break
            if mutant != "q_reload_early":
                yield ("wait", f"q_empty{c}", (k & 1) ^ 1)

            def q_issue(c=c):
                check(Qb[c] is None or s_done[c] >= last_s_of_unit.get((c, Qb[c]), -1),
                      f"Q buffer of set {c} reloaded before the last S of unit {Qb[c]}")
                Qb[c] = None

            def q_land(c=c, u=u):
                Qb[c] = u
            yield ("act", q_issue)
            yield ("async", f"q_full{c}", q_land)
            for j in range(units[u]):
                if mutant != "k_reload_early":
                    yield ("wait", f"k_empty{c}", (g & 1) ^ 1)
                if fresh:
                    while stores[c] > 0 and mutant != "store_not_waited":
                        yield ("spin",)

                def k_issue(c=c, g=g):
                    check(stores[c] == 0, f"K buffer of set {c} reloaded under a cache store")
                    check(s_done[c] >= g - 1, f"K buffer of set {c} reloaded before S of tile {g - 1}")
                    Kb[c] = None

                def k_land(c=c, g=g):
                    Kb[c] = g
                yield ("act", k_issue)
                yield ("async", f"k_full{c}", k_land)
                if mutant != "v_reload_early":
                    yield ("wait", f"pv_done{c}", (g & 1) ^ 1)

                def v_issue(c=c, g=g):
                    check(stores[c] == 0, f"V buffer of set {c} reloaded under a cache store")
                    check(pv_done_t[c] >= g - 1, f"V buffer of set {c} reloaded before P V of tile {g - 1}")
                    Vb[c] = None

                def v_land(c=c, g=g):
                    Vb[c] = g
                yield ("act", v_issue)
                yield ("async", f"v_full{c}", v_land)
                if fresh and j % 2 == 0:        # this unit owns some of its tiles: store them
                    yield ("wait", f"k_full{c}", g & 1)
                    yield ("wait", f"v_full{c}", g & 1)
                    stores[c] += 1

                    def store_done(c=c, g=g):
                        check(Kb[c] == g and Vb[c] == g, f"cache store of tile {g} read a reloaded buffer")
                        stores[c] -= 1
                    yield ("async", None, store_done)
                g += 1
            k += 1

    last_s_of_unit = {}

    # ---------------- MMA issuer for both sets ----------------
    def mma():
        st = [{"live": True, "fresh": True, "j": 0, "g": 0, "k": 0, "u": None} for _ in range(SETS)]

        def issue_s(c):
            z = st[c]
            if z["fresh"]:
                u = yield from next_unit(c, z["k"])
                if u < 0:
                    z["live"] = False
                    return False
                z["u"], z["j"], z["fresh"] = u, 0, False
                yield ("wait", f"q_full{c}", z["k"] & 1)
            g, u = z["g"], z["u"]
            yield ("wait", f"k_full{c}", g & 1)
            if mutant != "s_before_pv_done":
                yield ("wait", f"pv_done{c}", (g & 1) ^ 1)

            def s_act(c=c, g=g, u=u):
                check(Kb[c] == g, f"S of tile {g} reads another K tile")
                check(Qb[c] == u, f"S of unit {u} reads the Q tile of unit {Qb[c]}")
                check(pv_done_t[c] >= g - 1, f"S({g}) overwrites P({g - 1}) while P V reads it")

            def s_land(c=c, g=g):
                S[c] = ("S", g)
                P_writers[c] = set()
                s_done[c] = g
            yield ("act", s_act)
            yield ("async", f"s_full{c}", s_land)
            yield ("async", f"k_empty{c}", None)
            if z["j"] + 1 == units[u]:
                last_s_of_unit[(c, u)] = g
                yield ("async", f"q_empty{c}", None)
            return True

        def issue_pv(c):
            z = st[c]
            g, u, j = z["g"], z["u"], z["j"]
            if mutant != "pv_before_p":
                yield ("wait", f"p_full{c}", g & 1)
            yield ("wait", f"v_full{c}", g & 1)
            if j == 0 and z["k"] > 0 and mutant != "o_overwrite_early":
                yield ("wait", f"o_empty{c}", (z["k"] & 1) ^ 1)

            def pv_act(c=c, g=g, u=u, j=j):
                check(S[c] == ("P", g) and len(P_writers[c]) == warps, f"P V of tile {g} reads an unfinished P")
                check(Vb[c] == g, f"P V of tile {g} reads another V tile")
                if j == 0:
                    check(not O_readers[c], f"O of set {c} restarted while unit {O[c]} is read")
                    O[c] = u
                else:
                    check(O[c] == u, "P V into another unit's accumulator")
                pv_issued[c] = g

            def pv_land(c=c, g=g):
                pv_done_t[c] = g
            yield ("act", pv_act)
            yield ("async", f"pv_done{c}", pv_land)
            z["g"] += 1
            z["j"] += 1
            if z["j"] == units[u]:

                def o_land(c=c):
                    O_readers[c] = set(range(warps))
                yield ("async", f"o_full{c}", o_land)
                z["fresh"] = True
                z["k"] += 1

        pend = []
        for c in range(SETS):
            pend.append((yield from issue_s(c)))
        while any(pend):
            for c in range(SETS):
                if not pend[c]:
                    continue
                yield from issue_pv(c)
                pend[c] = yield from issue_s(c)

    # ---------------- softmax warp w of set c ----------------
    def softmax(c, w):
        g, k = 0, 0
        while True:
            u = yield from next_unit(c, k)
            if u < 0:
                break
            n = units[u]
            for j in range(n):
                yield ("wait", f"s_full{c}", g & 1)
                yield ("act", lambda c=c, g=g: check(S[c] in (("S", g), ("P", g)), f"softmax read {S[c]}, not S({g})"))
                if j > 0 and rng.random() < 0.3:   # the reference maximum moved: rescale O
                    yield ("act", lambda c=c, g=g: check(pv_done_t[c] >= g - 1 and pv_issued[c] == g - 1,
                                                         "O rescaled under a P V"))

                # the remainder vote: warp 0 clears the next tile's word, every warp ORs its
                # need into this tile's word, arrives, waits for the others, reads the answer
                need = rng.random() < 0.3
                if w == 0:
                    slot = (g + 1) % 3 if mutant != "vote_clear_wrong_word" else g % 3
                    yield ("act", lambda c=c, slot=slot: vote_word[c].__setitem__(slot, 0))

                def vote(c=c, g=g, need=need):
                    vote_need[c][g] = vote_need[c].get(g, False) or need
                    if need:
                        vote_word[c][g % 3] = 1
                yield ("act", vote)
                yield ("arrive", f"vote{c}")
                if mutant != "vote_not_waited":
                    yield ("wait", f"vote{c}", g & 1)

                def read_vote(c=c, g=g):
                    vote_seen[c].setdefault(g, []).append(vote_word[c][g % 3] != 0)
                yield ("act", read_vote)

                def p_write(c=c, g=g, w=w):
                    check(pv_done_t[c] >= g - 1, f"P({g}) written over P({g - 1}) while P V reads it")
                    S[c] = ("P", g)
                    P_writers[c].add(w)
                yield ("act", p_write)
                if j == n - 1 and rng.random() < 0.5:   # a ragged tile: zero the V rows past the end
                    if mutant != "zero_before_v_lands":
                        yield ("wait", f"v_full{c}", g & 1)
                    yield ("act", lambda c=c, g=g: check(Vb[c] == g, "zeroed rows of another V tile"))
                yield ("arrive", f"p_full{c}")
                g += 1
            if mutant != "o_read_early":
                yield ("wait", f"o_full{c}", k & 1)
            yield ("act", lambda c=c, u=u, w=w: check(O[c] == u and w in O_readers[c] and pv_done_t[c] == g - 1,
                                                      f"read O of unit {O[c]} before unit {u} was complete"))
            yield ("act", lambda c=c, w=w: O_readers[c].discard(w))
            yield ("arrive", f"o_empty{c}")
            if w == 0:
                units_done.append(u)
            k += 1

    roles = {"MMA": mma()}
    for c in range(SETS):
        roles[f"PR{c}"] = producer(c)
        for w in range(warps):
            roles[f"SM{c}.{w}"] = softmax(c, w)
    waiting = {r: None for r in roles}
    resume = {r: None for r in roles}
    done = set()
    pending = []                       # (issuer, seq, bar, callback)
    seq = 0
    for step in range(4_000_000):
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
    for c in range(SETS):
        for g, seen in vote_seen[c].items():
            check(all(v == vote_need[c][g] for v in seen), f"set {c} disagreed on the remainder of tile {g}")
    check(all(v == 0 for v in stores), "cache stores still in flight at the end")


def _workloads(n, seed):
    rng = random.Random(seed)
    return [[rng.choice([1, 1, 2, 3, 4, 7, 16]) for _ in range(rng.randint(1, 9))] for _ in range(n)]


@pytest.mark.parametrize("fresh", [False, True])
def test_schedule_has_no_race_and_no_deadlock(fresh):
    for i, units in enumerate(_workloads(300, 7 + fresh)):
        simulate(units, seed=i, fresh=fresh)


def test_schedule_with_four_softmax_warps_per_set():
    for i, units in enumerate(_workloads(60, 21)):
        simulate(units, seed=i, fresh=i % 2 == 1, warps=4)


@pytest.mark.parametrize("mutant,fresh", [
    ("k_reload_early", False),       # K(g) loaded before S(g-1) has read the buffer
    ("v_reload_early", False),       # V(g) loaded before P(g-1) V(g-1) has read the buffer
    ("q_reload_early", False),       # the next unit's Q loaded before this unit's last S
    ("s_before_pv_done", False),     # S(g) written over P(g-1) while P(g-1) V(g-1) reads it
    ("pv_before_p", False),          # P V issued before every warp has written P
    ("o_read_early", False),         # O read out before the unit's last P V completed
    ("zero_before_v_lands", False),  # V rows zeroed before the tile's load has landed
    ("vote_not_waited", False),      # the remainder vote read before every warp has voted
    ("vote_clear_wrong_word", False),  # warp 0 clears the word of the tile being voted on
    ("store_not_waited", True),      # a K/V buffer reloaded while a cache store still reads it
])
def test_planted_schedule_mistakes_are_caught(mutant, fresh):
    with pytest.raises(Race):
        for i, units in enumerate(_workloads(300, 11)):
            simulate(units, seed=i, fresh=fresh, mutant=mutant)
