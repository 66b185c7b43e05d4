"""Host-side model of the 64-row tcgen05 kernel's mbarrier protocol (csrc/decode_wide.cu).

The kernel's warps hand work to each other through shared-memory mbarriers that are waited
on by phase parity.  A parity wait is only meaningful while the barrier is at most one phase
ahead of the phase the waiter wants, and a barrier that counts several arrivals (the four
softmax warps) must not receive one warp's arrival for the next phase before another warp's
arrival for the current one.  This model runs the kernel's agents as coroutines with random
timings and checks, on every wait, that neither can happen, that every PV is issued only
after all four softmax warps published that group's P tile, and that the walk never
deadlocks:

- producer: pages in order through a three-slot ring (FULL / EMPTY per slot);
- MMA thread: the kernel's dynamic loop (PV first, QK of group g only after PV of g - 2),
  issuing into an in-order tensor pipe whose commits arrive when all earlier work is done;
  issuing blocks until the pipe has nearly drained, as on the hardware;
- four softmax warps, independent: score buffer A (page pairs) or B (single pages), P-ready
  barrier by group parity, PV-done wait only before a rescale, epilogue per piece;
- four query-loader warps: next piece's query tile after the previous piece's last QK.

The grouping rule (wide_group) and every barrier count follow the kernel.  No GPU is used.
"""

import heapq
import random

import pytest

NS = 3  # page ring depth


def wide_group(it, n, ntiles):
    """Pages in the score group starting at page n of a piece (it = CTA-wide page count)."""
    return 2 if (it % NS != NS - 1 and n + 1 < ntiles) else 1


class ProtocolError(AssertionError):
    pass


class Bar:
    """An mbarrier: `count` arrivals complete a phase.  Waits name the phase index they
    want; the parity test is checked against the one-phase window it relies on."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, k):
        if self.phase > k + 1:
            raise ProtocolError(f"{self.name}: waiting for phase {k} with {self.phase} completed (parity alias)")
        return (self.phase & 1) != (k & 1)


class Model:
    def __init__(self, pieces, rng, two_p_barriers=True, rescale_p=0.3):
        self.pieces, self.rng, self.two_p, self.rescale_p = pieces, rng, two_p_barriers, rescale_p
        self.now, self.events, self.seq = 0.0, [], 0
        self.pipe_free = 0.0
        b = {}
        for s in range(NS):
            b[("FULL", s)] = Bar(f"FULL{s}", 1)
            b[("EMPTY", s)] = Bar(f"EMPTY{s}", 1)
        b["QFULL"], b["QFREE"] = Bar("QFULL", 4), Bar("QFREE", 1)
        for i in range(2):
            b[("SFULL", i)] = Bar(f"SFULL{i}", 1)
            b[("SFREE", i)] = Bar(f"SFREE{i}", 4)
            b[("PFULL", i)] = Bar(f"PFULL{i}", 4)
            b[("PVDONE", i)] = Bar(f"PVDONE{i}", 1)
        b["OFULL"], b["OFREE"] = Bar("OFULL", 1), Bar("OFREE", 4)
        self.b = b
        self.published = {}  # group -> softmax warps that wrote their rows of P

    # ----- tensor pipe -----
    def mma(self, dur):
        self.pipe_free = max(self.now, self.pipe_free) + dur

    def commit(self, key):
        self.at(self.pipe_free + 1e-6, self.b[key].arrive)

    def at(self, t, fn):
        self.seq += 1
        heapq.heappush(self.events, (t, self.seq, fn))

    # ----- agents (generators yielding a predicate or ("sleep", dt)) -----
    def producer(self):
        it = 0
        for nt in self.pieces:
            for _ in range(nt):
                s, k = it % NS, it // NS
                if k > 0:
                    yield lambda s=s, k=k: self.b[("EMPTY", s)].done(k - 1)
                self.at(self.now + self.rng.expovariate(1 / 1.5), self.b[("FULL", s)].arrive)
                it += 1

    def loader(self):
        for j in range(len(self.pieces)):
            yield ("sleep", self.rng.uniform(0.0, 0.5))
            if j > 0:
                yield lambda j=j: self.b["QFREE"].done(j - 1)
            self.b["QFULL"].arrive()

    def softmax(self, w):
        it = g = 0
        uses = [0, 0]
        for j, nt in enumerate(self.pieces):
            n = 0
            while n < nt:
                gsz = wide_group(it, n, nt)
                sb = 0 if gsz == 2 else 1
                yield lambda sb=sb, u=uses[sb]: self.b[("SFULL", sb)].done(u)
                self.b[("SFREE", sb)].arrive()
                uses[sb] += 1
                yield ("sleep", self.rng.expovariate(1 / 0.8))
                if n > 0 and self.rng.random() < self.rescale_p:
                    # the kernel waits for the previous group's PV before rescaling O
                    yield lambda g=g: self.b[("PVDONE", (g - 1) & 1)].done((g - 1) >> 1)
                    yield ("sleep", 0.2)
                self.published[g] = self.published.get(g, 0) + 1
                self.b[("PFULL", g & 1 if self.two_p else 0)].arrive()
                g += 1
                n += gsz
                it += gsz
            yield lambda j=j: self.b["OFULL"].done(j)
            yield ("sleep", self.rng.expovariate(1.0))
            self.b["OFREE"].arrive()

    def pfull_ready(self, g):
        if self.two_p:
            return self.b[("PFULL", g & 1)].done(g >> 1)
        return self.b[("PFULL", 0)].done(g)

    def mma_thread(self):
        rng, b, pieces = self.rng, self.b, self.pieces
        qk = {"p": 0, "n": 0, "it": 0, "g": 0}
        pv = {"p": 0, "n": 0, "it": 0, "g": 0}
        uses = [0, 0]
        have_q = False
        while pv["p"] < len(pieces):
            progressed = False
            if pv["g"] < qk["g"]:
                nt = pieces[pv["p"]]
                gsz = wide_group(pv["it"], pv["n"], nt)
                first = pv["n"] == 0
                if self.pfull_ready(pv["g"]) and (not first or pv["p"] == 0 or b["OFREE"].done(pv["p"] - 1)):
                    if self.published.get(pv["g"], 0) != 4:
                        raise ProtocolError(f"PV of group {pv['g']} issued before all four P rows were written")
                    for j in range(gsz):
                        self.mma(rng.uniform(0.3, 0.7))
                        self.commit(("EMPTY", (pv["it"] + j) % NS))
                    self.commit(("PVDONE", pv["g"] & 1))
                    pv["n"] += gsz
                    pv["it"] += gsz
                    pv["g"] += 1
                    if pv["n"] == nt:
                        self.commit("OFULL")
                        pv["p"] += 1
                        pv["n"] = 0
                    progressed = True
            if not progressed and qk["p"] < len(pieces) and qk["g"] < pv["g"] + 2:
                if not have_q:
                    have_q = b["QFULL"].done(qk["p"])
                nt = pieces[qk["p"]]
                gsz = wide_group(qk["it"], qk["n"], nt)
                sb = 0 if gsz == 2 else 1
                landed = all(b[("FULL", (qk["it"] + k) % NS)].done((qk["it"] + k) // NS) for k in range(gsz))
                if have_q and landed and (uses[sb] == 0 or b[("SFREE", sb)].done(uses[sb] - 1)):
                    self.mma(rng.uniform(0.3, 2.0))
                    self.commit(("SFULL", sb))
                    uses[sb] += 1
                    qk["n"] += gsz
                    qk["it"] += gsz
                    qk["g"] += 1
                    if qk["n"] == nt:
                        self.commit("QFREE")
                        have_q = False
                        qk["p"] += 1
                        qk["n"] = 0
                    progressed = True
            if progressed:
                # issuing blocks until the pipe has taken all but its last instructions
                yield ("sleep", max(0.0, self.pipe_free - self.now - rng.uniform(0.05, 0.2)))
            else:
                yield ("poll",)

    # ----- scheduler -----
    def run(self):
        agents = {"producer": self.producer(), "mma": self.mma_thread()}
        for w in range(4):
            agents[f"softmax{w}"] = self.softmax(w)
            agents[f"loader{w}"] = self.loader()
        waiting, changed = {}, [True]

        def step(k):
            changed[0] = True
            try:
                w = next(agents[k])
            except StopIteration:
                waiting.pop(k, None)
                agents.pop(k)
                return
            if isinstance(w, tuple) and w[0] == "sleep":
                w = ("until", self.now + w[1])
            waiting[k] = w

        for k in list(agents):
            step(k)
        while agents:
            progressed = False
            for k in list(agents):
                w = waiting.get(k)
                if callable(w) and w():
                    step(k)
                    progressed = True
                elif isinstance(w, tuple) and w[0] == "until" and self.now >= w[1]:
                    step(k)
                    progressed = True
            if "mma" in agents and waiting.get("mma") == ("poll",) and changed[0]:
                changed[0] = False
                step("mma")
                progressed = progressed or waiting.get("mma") != ("poll",)
            if progressed:
                continue
            times = [w[1] for w in waiting.values() if isinstance(w, tuple) and w[0] == "until"]
            if self.events:
                times.append(self.events[0][0])
            if not times:
                stuck = sorted(k for k, w in waiting.items() if callable(w) or w == ("poll",))
                raise ProtocolError(f"deadlock: {stuck} wait for barriers no agent will complete")
            self.now = max(self.now, min(times))
            while self.events and self.events[0][0] <= self.now:
                heapq.heappop(self.events)[2]()
            changed[0] = True


def random_pieces(rng):
    return [rng.choice([1, 1, 2, 2, 3, 4, 5, 8, 16, 40]) for _ in range(rng.randint(1, 25))]


def test_group_rule_pairs_only_adjacent_slots_of_one_piece():
    it = 0
    for nt in [1, 2, 3, 4, 5, 7, 1, 2]:
        n = 0
        while n < nt:
            g = wide_group(it, n, nt)
            if g == 2:
                assert it % NS in (0, 1) and n + 1 < nt
            n += g
            it += g
        assert n == nt


def test_protocol_holds_under_random_timing():
    rng = random.Random(2024)
    for _ in range(60):
        Model(random_pieces(rng), rng).run()


def test_model_sees_the_race_of_a_single_p_barrier():
    # With one P-ready barrier a softmax warp that finished group g + 1 completes group g's
    # phase for a slower warp: the checks above must be able to see that.
    rng = random.Random(7)
    caught = 0
    for _ in range(30):
        try:
            Model(random_pieces(rng), rng, two_p_barriers=False).run()
        except ProtocolError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("pieces", [[1] * 12, [2] * 8, [5, 1, 1, 4, 2, 3], [40], [1, 40, 1]])
def test_protocol_on_fixed_piece_patterns(pieces):
    rng = random.Random(sum(pieces))
    for _ in range(10):
        Model(pieces, rng).run()
