"""Hand-off model of grouped_forward_kernel: deadlock, phase-aliasing and data-race check (CPU).

The head-group kernel's 16 warps meet only through mbarriers. This test runs a
model of one CTA: every role is a generator that performs, in the kernel's
order, its mbarrier waits and arrives, its asynchronous operations (TMA loads
and stores, tcgen05 products and their commits) and its reads and writes of
the shared-memory and tensor-memory buffers. A scheduler interleaves the roles
and completes asynchronous operations at random (in issue order per issuing
thread, as tcgen05 operations complete; each TMA load on its own), and:

- fails on a deadlock (no role can move and nothing is in flight);
- fails when a parity wait could be satisfied by a phase two ahead of the one
  it means (every wait names its phase);
- fails on a data race: two accesses to one buffer part, at least one a write,
  with neither ordered before the other. Order is happens-before through the
  mbarriers, tracked with vector clocks; an asynchronous operation's accesses
  are ordered after another access only through its own completion (the
  commit's or the TMA's arrival, or the wait for the store's read).

A negative control drops one wait of the kernel (the states issuer's wait for
its tile's C/B load, whose absence let the states product read a stale B) and
checks that the model reports the race.

The model is written from the kernel's role loops; it is a check of the
protocol, not of the arithmetic. Buffer parts: shared memory C, B, X (then X')
per stage, H' and the two tile records; tensor memory S (split into the tril
half and the exact form's S~ half), h and the two Z buffers; a part is a
32-row lane quadrant where the warps that touch it own one.
"""
import random

import pytest

KH = 2

# mbarrier indices (the kernel's, plus the model's own for asynchronous ops)
(FULL_CB, EMPTY_CB, FULL_X, EMPTY_X, XP_FULL, REC_FULL, REC_EMPTY, S_FULL, S_FREE, TRIL_FULL) = (
    0, 2, 4, 6, 8, 10, 12, 14, 16, 18)
(H_READY, HP_FULL, HP_EMPTY, STATES_DONE, Z_FULL) = (20, 21, 22, 23, 24)
(M3_DONE, Z_SCALED, RAW_X, SLOT_FULL, SLOT_FREE) = (26, 27, 28, 29, 30)
(PUB, Y_STAGED, Z_EMPTY, Z_INIT) = (42, 43, 44, 46)
NBARS = 48


def bar_count(i):
    if i in (EMPTY_CB, EMPTY_CB + 1):
        return 3
    if i in (EMPTY_X, EMPTY_X + 1):
        return 2
    if i in (REC_EMPTY, REC_EMPTY + 1):
        return 13
    if i in (TRIL_FULL, TRIL_FULL + 1, Z_EMPTY, Z_EMPTY + 1, SLOT_FULL, H_READY, HP_FULL, Z_SCALED, PUB,
             XP_FULL, XP_FULL + 1, Z_INIT, Z_INIT + 1, Y_STAGED):
        return 4
    return 1


ALL = (0, 1, 2, 3)


class Race(Exception):
    pass


class Stuck(Exception):
    pass


def vc_join(a, b):
    out = dict(a)
    for k, v in b.items():
        if out.get(k, 0) < v:
            out[k] = v
    return out


def vc_leq(a, b):
    return all(b.get(k, 0) >= v for k, v in a.items())


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0
        self.acc = {}        # clock joined over the arrivals of the current phase
        self.clocks = []     # clock of each completed phase

    def arrive(self, clock):
        self.acc = vc_join(self.acc, clock)
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.clocks.append(self.acc)
            self.acc, self.pending = {}, self.count
            self.phase += 1


# actions a role yields
def W(bar, parity, phase):          # wait; phase < 0: the barrier's initial phase (passes at once)
    return ("wait", bar, parity, phase)


def A(bar):                         # arrive
    return ("arrive", bar)


def R(*parts):                      # read buffer parts, e.g. R(("X", 0, q))
    return ("access", "r", parts)


def Wr(*parts):
    return ("access", "w", parts)


def ASYNC(queue, reads, writes, arrive=None):
    """An asynchronous operation on an in-order queue (a tcgen05 issuer, or a
    private queue per TMA load): it reads and writes at some later moment and
    then, if given, arrives on a barrier carrying its own event."""
    return ("async", queue, tuple(reads), tuple(writes), arrive)


def COMMIT(queue, *bars):           # tcgen05.commit: arrive once every earlier op of the queue is done
    return ("async", queue, (), (), bars)


def JOIN(queue):                    # wait until every op of the queue is done (the store's wait_group.read)
    return ("join", queue)


def parts(name, idx, quads=ALL):
    return [(name, idx, q) for q in quads]


class Model:
    """pieces: list of (first tile index within the chain, number of tiles, publishes at its end)."""

    def __init__(self, pieces, hard=frozenset(), states_waits_cb=True):
        self.tiles = []
        for pi, (t0, n, pub) in enumerate(pieces):
            for t in range(n):
                self.tiles.append(dict(piece=pi, first=t == 0, last=t == n - 1, pub=pub and t == n - 1,
                                       seed=t0 > 0 and t == 0))
        self.hard = hard
        self.states_waits_cb = states_waits_cb

    # ------------------------------------------------------------- roles
    def producer(self):
        for k, _ in enumerate(self.tiles):
            st, par = k & 1, (k >> 1) & 1
            yield W(EMPTY_X + st, par ^ 1, (k >> 1) - 1)
            yield ASYNC(("tmaX", k), [], parts("X", st), arrive=(FULL_X + st,))
            yield W(EMPTY_CB + st, par ^ 1, (k >> 1) - 1)
            yield ASYNC(("tmaCB", k), [], parts("C", st) + parts("B", st), arrive=(FULL_CB + st,))

    def prologue(self):
        for k, _ in enumerate(self.tiles):
            st, par = k & 1, (k >> 1) & 1
            yield W(REC_EMPTY + st, par ^ 1, (k >> 1) - 1)
            yield Wr(*parts("Rec", st))
            yield A(REC_FULL + st)

    def mma_z(self):
        q = "mmaZ"
        n = len(self.tiles)
        nh = 0

        def mma1(kk):
            s1 = kk & 1
            yield W(FULL_CB + s1, (kk >> 1) & 1, kk >> 1)
            if kk > 0:
                yield W(S_FREE, (kk - 1) & 1, kk - 1)
            yield ASYNC(q, parts("C", s1) + parts("B", s1), parts("Slo", 0) + parts("Shi", 0))
            yield COMMIT(q, S_FULL)

        if n:
            yield from mma1(0)
        for k in range(n):
            st, par = k & 1, (k >> 1) & 1
            hard = k in self.hard
            yield W(REC_FULL + st, par, k >> 1)
            yield R(*parts("Rec", st))
            yield A(REC_EMPTY + st)
            zb = k & 1
            yield W(HP_FULL, k & 1, k)
            yield W(Z_INIT + zb, (k >> 1) & 1, k >> 1)
            yield ASYNC(q, parts("C", st) + parts("Hp", 0) + parts("Z", zb), parts("Z", zb))
            if not hard:
                yield COMMIT(q, HP_EMPTY)
                yield W(TRIL_FULL + st, par, k >> 1)
                yield W(XP_FULL + st, par, k >> 1)
                yield ASYNC(q, parts("Slo", 0) + parts("X", st) + parts("Z", zb), parts("Z", zb))
                yield COMMIT(q, Z_FULL + zb, S_FREE)
            else:
                yield COMMIT(q, M3_DONE)
                yield W(M3_DONE, nh & 1, nh)
                yield ASYNC(("tmaRaw", k), [], parts("Hp", 0), arrive=(RAW_X,))
                yield W(RAW_X, nh & 1, nh)
                yield W(Z_SCALED, nh & 1, nh)
                for hh in range(KH):
                    u = nh * KH + hh
                    yield W(SLOT_FULL, u & 1, u)
                    yield ASYNC(q, parts("Shi", 0) + parts("Hp", 0) + parts("Z", zb), parts("Z", zb))
                    yield COMMIT(q, SLOT_FREE)
                yield COMMIT(q, Z_FULL + zb, S_FREE, HP_EMPTY)
                nh += 1
            yield COMMIT(q, EMPTY_CB + st, EMPTY_X + st)
            if k + 1 < n:
                yield from mma1(k + 1)

    def mma_s(self):
        q = "mmaS"
        for k, _ in enumerate(self.tiles):
            st, par = k & 1, (k >> 1) & 1
            if self.states_waits_cb:
                yield W(FULL_CB + st, par, k >> 1)
            yield W(XP_FULL + st, par, k >> 1)
            yield W(H_READY, k & 1, k)
            yield ASYNC(q, parts("B", st) + parts("X", st) + parts("H", 0), parts("H", 0))
            yield COMMIT(q, STATES_DONE, EMPTY_CB + st, EMPTY_X + st)

    def state(self, w):
        npub, nh = 0, 0
        mine = (w,)
        for k, tile in enumerate(self.tiles + [None]):
            if k >= 1:
                yield W(STATES_DONE, (k - 1) & 1, k - 1)
                prev = self.tiles[k - 1]
                if prev["last"]:
                    yield R(*parts("H", 0, mine))       # end state to the ring / final state
                    if prev["pub"]:
                        yield A(PUB)
                        if w == 0:
                            yield W(PUB, npub & 1, npub)
                        npub += 1
            if tile is None:
                break
            st, par = k & 1, (k >> 1) & 1
            hard = k in self.hard
            yield W(REC_FULL + st, par, k >> 1)
            yield R(*parts("Rec", st))
            yield W(HP_EMPTY, (k & 1) ^ 1, k - 1)
            if tile["first"]:
                yield Wr(*parts("H", 0, mine))          # the piece's starting state
            yield R(*parts("H", 0, mine))
            yield Wr(*parts("Hp", 0, mine), *parts("H", 0, mine))
            yield A(H_READY)
            yield A(HP_FULL)
            yield W(S_FULL, k & 1, k)
            yield R(*parts("Slo", 0, mine), *parts("Shi", 0, mine))
            yield Wr(*parts("Slo", 0, mine))
            yield A(TRIL_FULL + st)
            if hard:
                for hh in range(KH):
                    u = nh * KH + hh
                    yield W(SLOT_FREE, (u & 1) ^ 1, u - 1)
                    yield R(*parts("Slo", 0, mine))
                    yield Wr(*parts("Shi", 0, mine))
                    yield A(SLOT_FULL)
                nh += 1
            yield A(REC_EMPTY + st)

    def output(self, w):
        nh = 0
        mine = (w,)
        for k, _ in enumerate(self.tiles):
            st, par = k & 1, (k >> 1) & 1
            hard = k in self.hard
            yield W(REC_FULL + st, par, k >> 1)
            yield R(*parts("Rec", st))
            yield A(REC_EMPTY + st)
            zb = k & 1
            if hard:
                yield W(M3_DONE, nh & 1, nh)
                yield R(*parts("Z", zb, mine))
                yield Wr(*parts("Z", zb, mine))
                yield A(Z_SCALED)
                nh += 1
            yield W(Z_FULL + zb, (k >> 1) & 1, k >> 1)
            yield R(*parts("Z", zb, mine))
            yield A(Z_EMPTY + zb)
            yield Wr(*parts("C", st, mine))                 # y staged in the dead C buffer
            yield A(Y_STAGED)
            if w == 0:
                yield W(Y_STAGED, k & 1, k)
                yield ASYNC(("tmaY", k), parts("C", st), [])
                yield JOIN(("tmaY", k))
                yield A(EMPTY_CB + st)

    def scale(self, w):
        mine = (w,)
        for k, _ in enumerate(self.tiles):
            st, par = k & 1, (k >> 1) & 1
            yield W(REC_FULL + st, par, k >> 1)
            yield R(*parts("Rec", st))
            yield A(REC_EMPTY + st)
            zb = k & 1
            yield W(Z_EMPTY + zb, ((k >> 1) & 1) ^ 1, (k >> 1) - 1)
            yield W(FULL_X + st, par, k >> 1)
            yield R(*parts("X", st, mine))
            yield Wr(*parts("X", st, mine), *parts("Z", zb, mine))
            yield A(XP_FULL + st)
            yield A(Z_INIT + zb)

    def roles(self):
        out = [("prod", self.producer()), ("pro", self.prologue()), ("mmaZ", self.mma_z()),
               ("mmaS", self.mma_s())]
        for w in range(4):
            out += [(f"state{w}", self.state(w)), (f"out{w}", self.output(w)), (f"scale{w}", self.scale(w))]
        return out


def run(model, seed, slow=None, max_steps=200000):
    """Interleave the roles; raise Race / Stuck, or return the number of steps."""
    rng = random.Random(seed)
    bars = [Barrier(bar_count(i)) for i in range(NBARS)]
    clocks = {}                  # thread -> vector clock
    history = {}                 # buffer part -> list of (kind, clock, who)
    queues = {}                  # async queue -> list of pending ops (kind, reads, writes, arrive, clock)
    issuer_of = {}               # async queue -> issuing thread (for JOIN)
    roles = model.roles()
    state = {name: [gen, None] for name, gen in roles}
    for name, _ in roles:
        clocks[name] = {name: 1}
    done = set()
    event = [0]

    def tick(who):
        c = dict(clocks[who])
        c[who] = c.get(who, 0) + 1
        clocks[who] = c

    def access(kind, parts_, clock, who):
        for p in parts_:
            for k2, c2, who2 in history.get(p, ()):
                if (kind == "w" or k2 == "w") and not vc_leq(c2, clock) and who2 != who:
                    raise Race(f"{who} {kind} {p} vs {who2} {k2}")
            history.setdefault(p, []).append((kind, clock, who))

    def step_async(q):
        kind, reads, writes, arrive, clock = queues[q].pop(0)
        event[0] += 1
        # in-order completion: an operation is ordered after the ones issued
        # before it on the same queue
        own = vc_join(vc_join(clock, last_own.get(q, {})), {("async", event[0]): 1})
        last_own[q] = own
        who = f"{q}"
        if reads:
            access("r", reads, own, who)
        if writes:
            access("w", writes, own, who)
        for b in arrive or ():
            bars[b].arrive(own)
        if not queues[q]:
            del queues[q]
        # what a JOIN on this queue will see
        joined_clock[q] = vc_join(joined_clock.get(q, {}), own)

    joined_clock = {}
    last_own = {}
    for name, _ in roles:
        state[name][1] = next(state[name][0])
    steps = 0
    force = False
    while len(done) < len(roles) or queues:
        progressed = held = False
        names = [n for n, _ in roles if n not in done]
        rng.shuffle(names)
        # complete some asynchronous operations (each queue in issue order)
        for q in list(queues):
            if rng.random() < 0.3:
                step_async(q)
                progressed = True
        for name in names:
            if slow and not force and name in slow and rng.random() < slow[name]:
                held = True  # held back this round; tried again before declaring a deadlock
                continue
            gen, act = state[name]
            ok = False
            if act[0] == "wait":
                _, b, parity, phase = act
                bar = bars[b]
                if phase >= 0 and bar.phase >= phase + 2:
                    raise Stuck(f"{name} waits for phase {phase} of barrier {b}, {bar.phase} completed")
                if parity != (bar.phase & 1):
                    ok = True
                    if phase >= 0:
                        assert bar.phase == phase + 1
                        clocks[name] = vc_join(clocks[name], bar.clocks[phase])
            elif act[0] == "arrive":
                tick(name)
                bars[act[1]].arrive(clocks[name])
                ok = True
            elif act[0] == "access":
                tick(name)
                access(act[1], act[2], clocks[name], name)
                ok = True
            elif act[0] == "async":
                _, q, reads, writes, arrive = act
                tick(name)
                queues.setdefault(q, []).append(("op", reads, writes, arrive, clocks[name]))
                issuer_of[q] = name
                ok = True
            elif act[0] == "join":
                q = act[1]
                if q not in queues:
                    clocks[name] = vc_join(clocks[name], joined_clock.get(q, {}))
                    ok = True
            if ok:
                progressed = True
                steps += 1
                try:
                    state[name][1] = next(gen)
                except StopIteration:
                    done.add(name)
        if not progressed and held and not force:
            force = True  # only held-back roles might move: let them
            continue
        force = False
        if not progressed and queues:
            step_async(rng.choice(sorted(queues, key=str)))  # only the hardware can move
            progressed = True
        if not progressed:
            blocked = {n: state[n][1] for n, _ in roles if n not in done}
            raise Stuck(f"deadlock: {blocked}")
        if steps > max_steps:
            raise Stuck("step limit")
    return steps


CASES = [
    dict(pieces=[(0, 3, False)]),                                      # one piece, ends the chain
    dict(pieces=[(0, 5, True), (0, 4, False)]),                        # head piece that publishes, then a chain
    dict(pieces=[(0, 2, True), (0, 6, False), (4, 3, False)]),          # wrap order: head, chain, tail
    dict(pieces=[(0, 6, False)], hard=frozenset({1, 2})),               # exact-form tiles in a row
    dict(pieces=[(0, 3, True), (2, 4, False)], hard=frozenset({0, 4})),  # exact form at piece starts
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_handoffs_are_race_and_deadlock_free(case):
    c = CASES[case]
    model = Model(c["pieces"], c.get("hard", frozenset()))
    for seed in range(12):
        run(model, seed)
    # one role at a time much slower than the rest
    for slow in ("prod", "pro", "mmaZ", "mmaS", "state3", "out0", "scale2"):
        run(model, 100 + case, slow={slow: 0.95})


def test_model_catches_the_states_product_reading_an_unloaded_b():
    # the kernel once lacked this wait: the states product could read the C/B
    # stage before its TMA load had landed
    model = Model([(0, 6, False)], states_waits_cb=False)
    caught = 0
    for seed in range(40):
        try:
            run(model, seed, slow={"prod": 0.6})
        except Race as e:
            assert "B" in str(e)
            caught += 1
    assert caught > 0
