"""Race check, on the CPU, of the multi-token decode kernel's barrier protocol.

k_verify_tc runs four roles: a TMA producer, an MMA issuer, the softmax
warps (modelled as one agent: they pass the same named barriers together)
and, asynchronously, the tensor pipe and the copy engine. This test models
them step by step as the kernel orders them, with mbarriers that behave as
the hardware's do: a phase completes when its arrivals are in, and a wait on
a parity returns as soon as the barrier's current phase has the other
parity. A wait is correct only if it returns exactly when the phase it means
has completed; the model flags any wait that returns early or misses its
phase (parity aliasing), and any access to shared memory or TMEM that an
in-flight copy or MMA could still touch. A random scheduler interleaves the
roles over many seeds.

With one P-ready barrier for both shared-memory P buffers the checker finds
schedules where the softmax arrives for tile j before the issuer has waited
for tile j - 1; with one barrier per buffer (the kernel's protocol) it finds
no violation and no deadlock."""
from __future__ import annotations

import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


class Model:
    """One CTA of the kernel: n_tiles key tiles, MT 128-dim blocks of K and V
    per tile, an NSTAGE ring; rescale decisions drawn at random."""

    def __init__(self, n_tiles, MT, NSTAGE, per_buffer_p_ready, rng, skip=()):
        self.n, self.MT, self.NS, self.rng = n_tiles, MT, NSTAGE, rng
        self.per_buffer = per_buffer_p_ready
        self.skip = set(skip)  # waits left out, to show the checker catches their absence
        B = Bar
        self.q_full = B("q_full", 1)
        self.full = [B("full%d" % s, 1) for s in range(NSTAGE)]
        self.empty = [B("empty%d" % s, 1) for s in range(NSTAGE)]
        self.s_full = [B("s_full0", 1), B("s_full1", 1)]
        self.o_done = [B("o_done0", 1), B("o_done1", 1)]
        self.p_ready = [B("p_ready0", 1), B("p_ready1", 1)] if per_buffer_p_ready else [B("p_ready", 1)]
        self.violations = []
        # asynchronous engines
        self.tc_queue = []          # ("mma", tag, reads, writes) or ("commit", bar), in issue order
        self.tma_inflight = []      # (stage, bar)
        # state for hazard checks
        self.s_read = set()         # tiles whose S the softmax has read
        self.s_done = set()         # tiles whose S MMAs completed
        self.p_written = set()      # tiles whose P the softmax has written
        self.pv_done = set()        # tiles whose PV completed (all MT blocks)
        self.pv_parts = {}

    # ---------------------------------------------------------------- helpers
    def check_wait(self, bar, k, role=None):
        """Hardware answer of a parity wait for phase k, checked against the
        truth (phase k complete)."""
        if role in self.skip:
            return True
        ret = (bar.phase & 1) != (k & 1)
        truth = bar.phase > k
        if ret != truth:
            self.violations.append("%s: wait for phase %d at phase %d returns %s" % (bar.name, k, bar.phase, ret))
        return ret

    def inflight_mma(self, pred):
        return any(op[0] == "mma" and pred(op) for op in self.tc_queue)

    def hazard(self, what):
        self.violations.append(what)

    # ---------------------------------------------------------------- roles
    def producer(self):
        self.tma_inflight.append(("Q", self.q_full))
        item = 0
        for j in range(self.n + 1):
            for kind in (0, 1):
                if (kind == 0 and j == self.n) or (kind == 1 and j == 0):
                    continue
                for _ in range(self.MT):
                    s = item % self.NS
                    if item >= self.NS:
                        k = item // self.NS - 1
                        while not self.check_wait(self.empty[s], k, "empty"):
                            yield
                    if self.inflight_mma(lambda op: ("stage", s) in op[2]):
                        self.hazard("TMA into stage %d while an MMA reads it" % s)
                    self.tma_inflight.append((("stage", s), self.full[s]))
                    item += 1
                    yield

    def issuer(self):
        while not self.check_wait(self.q_full, 0):
            yield
        item = 0
        for j in range(self.n + 1):
            if j < self.n:
                if j >= 2 and (j - 2) not in self.s_read:
                    self.hazard("S_%d issued into the buffer of S_%d before the softmax read it" % (j, j - 2))
                for _ in range(self.MT):
                    s = item % self.NS
                    while not self.check_wait(self.full[s], item // self.NS):
                        yield
                    self.tc_queue.append(("mma", ("S", j), {("stage", s), "Q"}, {("S", j & 1)}))
                    self.tc_queue.append(("commit", self.empty[s]))
                    item += 1
                    yield
                self.tc_queue.append(("commit", self.s_full[j & 1], ("S", j)))
                yield  # nothing orders the issuer's next wait after this commit
            if j >= 1:
                t = j - 1
                bar, k = (self.p_ready[t & 1], t >> 1) if self.per_buffer else (self.p_ready[0], t)
                while not self.check_wait(bar, k, "p_ready"):
                    yield
                if t not in self.p_written:
                    self.hazard("PV_%d issued before P_%d was written" % (t, t))
                for _ in range(self.MT):
                    s = item % self.NS
                    while not self.check_wait(self.full[s], item // self.NS):
                        yield
                    self.tc_queue.append(("mma", ("PV", t), {("stage", s), ("P", t & 1)}, {"O"}))
                    self.tc_queue.append(("commit", self.empty[s]))
                    item += 1
                    yield
                self.tc_queue.append(("commit", self.o_done[t & 1], ("PV", t)))

    def softmax(self):
        pv_seen = 0
        for j in range(self.n):
            while not self.check_wait(self.s_full[j & 1], j >> 1, "s_full"):
                yield
            if j not in self.s_done:
                self.hazard("S_%d read before its MMA completed" % j)
            self.s_read.add(j)
            yield
            if j >= 1 and self.rng.random() < 0.4:  # a column maximum moved: rescale O
                if pv_seen < j:
                    while not self.check_wait(self.o_done[(j - 1) & 1], (j - 1) >> 1, "rescale"):
                        yield
                    pv_seen = j
                if self.inflight_mma(lambda op: "O" in op[3]):
                    self.hazard("O rescaled while a PV product is in flight (tile %d)" % j)
                yield
            if j >= 2 and pv_seen < j - 1:
                while not self.check_wait(self.o_done[j & 1], (j - 2) >> 1):
                    yield
                pv_seen = j - 1
            if self.inflight_mma(lambda op: ("P", j & 1) in op[2]):
                self.hazard("P_%d written while PV_%d reads the buffer" % (j, j - 2))
            if j >= 2 and (j - 2) not in self.pv_done:
                self.hazard("P_%d written before PV_%d completed" % (j, j - 2))
            self.p_written.add(j)
            (self.p_ready[j & 1] if self.per_buffer else self.p_ready[0]).arrive()
            yield
        t = self.n - 1
        while not self.check_wait(self.o_done[t & 1], t >> 1, "epilogue"):
            yield
        if self.inflight_mma(lambda op: "O" in op[3]):
            self.hazard("epilogue read O with a PV product in flight")

    def tensor_pipe_step(self):
        op = self.tc_queue.pop(0)
        if op[0] == "mma":
            tag = op[1]
            if tag[0] == "PV":
                self.pv_parts[tag[1]] = self.pv_parts.get(tag[1], 0) + 1
        else:  # commit: arrives once every earlier MMA has completed (they have: in order)
            if len(op) > 2:
                kind, t = op[2]
                if kind == "S":
                    self.s_done.add(t)
                elif self.pv_parts.get(t) == self.MT:
                    self.pv_done.add(t)
            op[1].arrive()

    def copy_engine_step(self):
        i = self.rng.randrange(len(self.tma_inflight))
        _, bar = self.tma_inflight.pop(i)
        bar.arrive()

    def run(self, max_steps=100000):
        agents = {"producer": self.producer(), "issuer": self.issuer(), "softmax": self.softmax()}
        done = set()
        for _ in range(max_steps):
            choices = [a for a in agents if a not in done]
            if self.tc_queue:
                choices.append("tc")
            if self.tma_inflight:
                choices.append("tma")
            if not choices:
                return
            c = self.rng.choice(choices)
            if c == "tc":
                self.tensor_pipe_step()
            elif c == "tma":
                self.copy_engine_step()
            else:
                try:
                    next(agents[c])
                except StopIteration:
                    done.add(c)
        # the roles only spin on waits, so running out of steps is a deadlock
        self.violations.append("deadlock: %s still running" % sorted(set(agents) - done))


CONFIGS = [(1, 1, 2), (2, 1, 2), (3, 2, 3), (5, 4, 5), (6, 2, 4), (8, 1, 3), (7, 4, 4)]


@pytest.mark.parametrize("n_tiles,MT,NSTAGE", CONFIGS)
def test_per_buffer_p_ready_has_no_race(n_tiles, MT, NSTAGE):
    for seed in range(300):
        m = Model(n_tiles, MT, NSTAGE, per_buffer_p_ready=True, rng=random.Random(seed))
        m.run()
        assert not m.violations, "seed %d: %s" % (seed, m.violations[:3])


def test_single_p_ready_barrier_can_alias():
    """The checker is not vacuous: with one barrier for both P buffers some
    schedule lets the softmax complete tile j's phase before the issuer
    waits for tile j - 1, and that wait then misses its phase."""
    found = []
    for seed in range(3000):
        m = Model(6, 1, 3, per_buffer_p_ready=False, rng=random.Random(seed))
        m.run()
        found += [v for v in m.violations if v.startswith("p_ready")]
        if found:
            break
    assert found, "no aliasing schedule found"
    assert "returns False" in found[0]


@pytest.mark.parametrize("wait", ["empty", "s_full", "p_ready", "rescale", "epilogue"])
def test_each_wait_is_needed(wait):
    """Leaving out any one of these waits lets some schedule touch a buffer an
    in-flight copy or MMA still uses (or deadlocks): the checks have teeth.
    (The softmax's wait for PV_{j-2} before it reuses a P buffer is not in
    the list: tcgen05 MMAs from one thread complete in order, so the S_j
    commit that starts tile j already follows PV_{j-2}.)"""
    for seed in range(400):
        m = Model(6, 2, 3, per_buffer_p_ready=True, rng=random.Random(seed), skip={wait})
        m.run()
        if m.violations:
            return
    pytest.fail("no schedule exposed the missing %s wait" % wait)
