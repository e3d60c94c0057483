"""Race check, on the CPU, of the attention kernels' barrier protocols.

Each tensor-core kernel runs four roles: a TMA producer, an MMA issuer, the
softmax warps (modelled as one agent per CTA: they pass the same barriers
together) and, asynchronously, the tensor pipe and the copy engine. This test
models them step by step as the kernels order them, with mbarriers that
behave as the hardware's do: a phase completes when its arrivals (and, for a
copy, its bytes) are in, and a wait on a parity returns as soon as the
barrier's current phase has the other parity. A wait is correct only if it
returns exactly when the phase it means has completed; the model flags any
wait that returns early or misses its phase (parity aliasing), any access to
shared memory or TMEM that an in-flight copy or MMA could still touch, and
deadlock. The tensor pipe completes one thread's MMAs in issue order, and a
commit arrives once every earlier MMA has completed. A random scheduler
interleaves the roles over many seeds.

Kernels modelled:
- k_verify_tc (multi-token decode): P^T in two shared-memory buffers, one
  P-ready barrier per buffer. With a single barrier for both, the checker
  finds schedules where the softmax arrives for tile j before the issuer
  has waited for tile j - 1.
- k_prefill_tc: P written over S in TMEM, one P-ready barrier; the softmax
  consumes PV_{j-1} before it arrives for tile j.
- k_prefill_pair: two CTAs; both producers fill their halves of a stage,
  which complete on the leader's barrier (armed by the leader for both
  halves' bytes); the leader issues cta_group::2 MMAs that read both CTAs'
  shared memory and write both TMEMs; commits arrive on both CTAs'
  barriers; both CTAs' softmax warps arrive on the leader's P-ready barrier.
- k_decode_split / k_decode_split_q8: a copy warp fills a ring of slots that
  three consumer warps take in turn; the ring size must be a multiple of the
  consumer count (which the kernels assert), else a parity wait can return
  for a slot's previous fill.
- k_verify_tc's failure paths, one agent per warp: bounded waits give up at
  random points; every warp still reaches the end, the four softmax warps
  together (their decisions that lead to a named barrier are votes), TMEM is
  released only after the MMAs drain, and no copy is in flight at exit.
"""
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


KERNELS = {
    # CTAs, P in shared memory (else over S in TMEM), one P-ready barrier per
    # P buffer, the softmax consumes PV_{j-1} before it arrives for tile j
    "verify": dict(n_cta=1, smem_p=True, per_buffer=True, pv_before_arrive=False),
    "verify_single_p_ready": dict(n_cta=1, smem_p=True, per_buffer=False, pv_before_arrive=False),
    "prefill": dict(n_cta=1, smem_p=False, per_buffer=False, pv_before_arrive=True),
    "pair": dict(n_cta=2, smem_p=False, per_buffer=False, pv_before_arrive=True),
}


class Model:
    """One CTA (or CTA pair) of a kernel over n_tiles key tiles, with KS
    stages of K and VS stages of V per tile through an NSTAGE ring;
    rescale decisions drawn at random."""

    def __init__(self, kernel, n_tiles, KS, VS, NSTAGE, rng, skip=()):
        cfg = KERNELS[kernel]
        self.C = cfg["n_cta"]
        self.smem_p, self.per_buffer = cfg["smem_p"], cfg["per_buffer"]
        self.pv_before_arrive = cfg["pv_before_arrive"]
        self.n, self.KS, self.VS, self.NS, self.rng = n_tiles, KS, VS, NSTAGE, rng
        self.skip = set(skip)  # waits left out, to show the checker catches their absence
        C, B = self.C, Bar
        arms = 1 + C if C > 1 else 1  # pair: the leader's arm and both halves' bytes
        self.q_full = B("q_full", arms)
        self.full = [B("full%d" % s, arms) for s in range(NSTAGE)]  # the leader's
        self.empty = [[B("empty%d/cta%d" % (s, c), 1) for s in range(NSTAGE)] for c in range(C)]
        self.s_full = [[B("s_full%d/cta%d" % (i, c), 1) for i in range(2)] for c in range(C)]
        self.o_done = [[B("o_done%d/cta%d" % (i, c), 1) for i in range(2)] for c in range(C)]
        self.p_ready = [B("p_ready%d" % i, C) for i in range(2 if self.per_buffer else 1)]
        self.violations = []
        self.tc_queue = []      # ("mma", tag, reads, writes) or ("commit", [bars], done-tag), issue order
        self.tma_inflight = []  # (resource written, bar)
        self.s_read = [set() for _ in range(C)]
        self.s_done, self.pv_done, self.pv_parts = set(), set(), {}
        self.p_written = [set() for _ in range(C)]

    # ---------------------------------------------------------------- helpers
    def check_wait(self, bar, k, role=None):
        """Hardware answer of a parity wait for phase k, checked against the
        truth (phase k complete)."""
        if role in self.skip:
            return True
        ret = (bar.phase & 1) != (k & 1)
        if ret != (bar.phase > k):
            self.violations.append("%s: wait for phase %d at phase %d returns %s" % (bar.name, k, bar.phase, ret))
        return ret

    def inflight(self, pred):
        return any(op[0] == "mma" and pred(op) for op in self.tc_queue)

    def reads(self, res):
        return self.inflight(lambda op: res in op[2])

    def writes(self, res):
        return self.inflight(lambda op: res in op[3])

    def hazard(self, what):
        self.violations.append(what)

    def p_res(self, c, t):
        return ("P", c, t & 1) if self.smem_p else ("S", c, t & 1)

    # ---------------------------------------------------------------- roles
    def producer(self, c):
        leader = c == 0
        if leader and self.C > 1:
            self.q_full.arrive()  # arm for both halves
        self.tma_inflight.append((("Q", c), self.q_full))
        item = 0
        for j in range(self.n + 1):
            for kind in (0, 1):
                if (kind == 0 and j == self.n) or (kind == 1 and j == 0):
                    continue
                for _ in range(self.KS if kind == 0 else self.VS):
                    s = item % self.NS
                    if item >= self.NS:
                        while not self.check_wait(self.empty[c][s], item // self.NS - 1, "empty"):
                            yield
                    if self.reads(("stage", c, s)):
                        self.hazard("copy into stage %d of CTA %d while an MMA reads it" % (s, c))
                    if leader and self.C > 1:
                        self.full[s].arrive()  # arm
                    self.tma_inflight.append((("stage", c, s), self.full[s]))
                    item += 1
                    yield

    def issuer(self):
        C = range(self.C)
        while not self.check_wait(self.q_full, 0, "q_full"):
            yield
        item = 0
        for j in range(self.n + 1):
            if j < self.n:
                for c in C:
                    if j >= 2 and (j - 2) not in self.s_read[c]:
                        self.hazard("S_%d issued over S_%d before CTA %d read it" % (j, j - 2, c))
                for _ in range(self.KS):
                    s = item % self.NS
                    while not self.check_wait(self.full[s], item // self.NS, "full"):
                        yield
                    self.tc_queue.append(("mma", ("S", j), {("stage", c, s) for c in C} | {("Q", c) for c in C},
                                          {("S", c, j & 1) for c in C}))
                    self.tc_queue.append(("commit", [self.empty[c][s] for c in C], None))
                    item += 1
                    yield
                self.tc_queue.append(("commit", [self.s_full[c][j & 1] for c in C], ("S", j)))
                yield  # nothing orders the issuer's next wait after this commit
            if j >= 1:
                t = j - 1
                bar, k = (self.p_ready[t & 1], t >> 1) if self.per_buffer else (self.p_ready[0], t)
                while not self.check_wait(bar, k, "p_ready"):
                    yield
                for c in C:
                    if t not in self.p_written[c]:
                        self.hazard("PV_%d issued before CTA %d wrote P_%d" % (t, c, t))
                for _ in range(self.VS):
                    s = item % self.NS
                    while not self.check_wait(self.full[s], item // self.NS, "full"):
                        yield
                    self.tc_queue.append(("mma", ("PV", t),
                                          {("stage", c, s) for c in C} | {self.p_res(c, t) for c in C},
                                          {("O", c) for c in C}))
                    self.tc_queue.append(("commit", [self.empty[c][s] for c in C], None))
                    item += 1
                    yield
                self.tc_queue.append(("commit", [self.o_done[c][t & 1] for c in C], ("PV", t)))

    def softmax(self, c):
        pv_seen = 0

        def wait_pv(t, role):
            while not self.check_wait(self.o_done[c][t & 1], t >> 1, role):
                yield

        for j in range(self.n):
            while not self.check_wait(self.s_full[c][j & 1], j >> 1, "s_full"):
                yield
            if j not in self.s_done or self.writes(("S", c, j & 1)):
                self.hazard("CTA %d read S_%d with its MMA not complete" % (c, j))
            self.s_read[c].add(j)
            yield
            if j >= 1 and self.rng.random() < 0.4:  # a row or column maximum moved: rescale O
                if pv_seen < j:
                    yield from wait_pv(j - 1, "rescale")
                    pv_seen = j
                if self.writes(("O", c)) or self.reads(("O", c)):
                    self.hazard("CTA %d rescaled O with a PV product in flight (tile %d)" % (c, j))
                yield
            if self.smem_p and j >= 2 and pv_seen < j - 1:  # the shared-memory P buffer is free
                yield from wait_pv(j - 2, "p_buffer")
                pv_seen = j - 1
            res = self.p_res(c, j)
            if self.reads(res) or self.writes(res):
                self.hazard("CTA %d wrote P_%d over a buffer an MMA still uses" % (c, j))
            self.p_written[c].add(j)
            if self.pv_before_arrive and j >= 1 and pv_seen < j:
                yield from wait_pv(j - 1, "pv_before_arrive")
                pv_seen = j
            (self.p_ready[j & 1] if self.per_buffer else self.p_ready[0]).arrive()
            yield
        yield from wait_pv(self.n - 1, "epilogue")
        if self.writes(("O", c)):
            self.hazard("CTA %d read O in the epilogue with a PV product in flight" % c)

    def tensor_pipe_step(self):
        op = self.tc_queue.pop(0)
        if op[0] == "mma":
            if op[1][0] == "PV":
                self.pv_parts[op[1][1]] = self.pv_parts.get(op[1][1], 0) + 1
            return
        done = op[2]
        if done and done[0] == "S":
            self.s_done.add(done[1])
        elif done and self.pv_parts.get(done[1]) == self.VS:
            self.pv_done.add(done[1])
        for bar in op[1]:
            bar.arrive()

    def copy_engine_step(self):
        _, bar = self.tma_inflight.pop(self.rng.randrange(len(self.tma_inflight)))
        bar.arrive()

    def run(self, max_steps=200000):
        agents = {"issuer": self.issuer()}
        for c in range(self.C):
            agents["producer%d" % c] = self.producer(c)
            agents["softmax%d" % c] = self.softmax(c)
        done = set()
        for _ in range(max_steps):
            choices = [a for a in agents if a not in done]
            if self.tc_queue:
                choices.append("tc")
            if self.tma_inflight:
                choices.append("tma")
            if not choices:
                return
            pick = self.rng.choice(choices)
            if pick == "tc":
                self.tensor_pipe_step()
            elif pick == "tma":
                self.copy_engine_step()
            else:
                try:
                    next(agents[pick])
                except StopIteration:
                    done.add(pick)
        # the roles only spin on waits, so running out of steps is a deadlock
        self.violations.append("deadlock: %s still running" % sorted(set(agents) - done))


# (n_tiles, K stages per tile, V stages per tile, ring stages) as the kernels
# are configured -- multi-token: D / 128 of each; prefill head_dim 256: 2 K
# and 2 V stages of a 5-stage ring; pair head_dim 512: 2 K stages and 1 V
# stage of a 3-stage ring -- and shorter rings, to stress their reuse
SHAPES = {
    "verify": [(1, 1, 1, 2), (2, 2, 2, 3), (3, 2, 2, 5), (6, 4, 4, 5), (8, 1, 1, 3), (7, 4, 4, 4)],
    "prefill": [(1, 2, 2, 5), (3, 2, 2, 5), (6, 2, 2, 5), (9, 2, 2, 4), (5, 4, 2, 3)],
    "pair": [(1, 2, 1, 3), (4, 2, 1, 3), (7, 2, 1, 3), (6, 1, 1, 2), (5, 2, 1, 4)],
}


@pytest.mark.parametrize("kernel,shape", [(k, s) for k, ss in SHAPES.items() for s in ss])
def test_kernel_protocol_has_no_race(kernel, shape):
    for seed in range(250):
        m = Model(kernel, *shape, rng=random.Random(seed))
        m.run()
        assert not m.violations, "%s %s seed %d: %s" % (kernel, shape, seed, m.violations[:3])


def test_single_p_ready_barrier_with_two_smem_buffers_can_alias():
    """The checker is not vacuous: with one barrier for both shared-memory P
    buffers (and no wait for PV_{j-1} before arriving) some schedule lets
    the softmax complete tile j's phase before the issuer waits for tile
    j - 1, and that wait then misses its phase."""
    found = []
    for seed in range(3000):
        m = Model("verify_single_p_ready", 6, 1, 1, 3, rng=random.Random(seed))
        m.run()
        found += [v for v in m.violations if v.startswith("p_ready")]
        if found:
            break
    assert found, "no aliasing schedule found"
    assert "returns False" in found[0]


@pytest.mark.parametrize("kernel,wait", [
    ("verify", "empty"), ("verify", "full"), ("verify", "s_full"), ("verify", "p_ready"),
    ("verify", "rescale"), ("verify", "epilogue"),
    ("prefill", "empty"), ("prefill", "s_full"), ("prefill", "p_ready"), ("prefill", "rescale"),
    ("prefill", "pv_before_arrive"), ("prefill", "epilogue"),
    ("pair", "empty"), ("pair", "full"), ("pair", "s_full"), ("pair", "p_ready"), ("pair", "rescale"),
    ("pair", "pv_before_arrive"), ("pair", "epilogue")])
def test_each_wait_is_needed(kernel, wait):
    """Leaving out any one of these waits lets some schedule touch a buffer an
    in-flight copy or MMA still uses, alias a parity wait or deadlock: the
    checks have teeth."""
    shape = {"verify": (6, 2, 2, 3), "prefill": (6, 2, 2, 3), "pair": (6, 2, 1, 3)}[kernel]
    for seed in range(600):
        m = Model(kernel, *shape, rng=random.Random(seed), skip={wait})
        m.run()
        if m.violations:
            return
    pytest.fail("no schedule exposed the missing %s wait in %s" % (wait, kernel))


def test_multi_token_p_buffer_wait_is_implied_by_in_order_completion():
    """The multi-token kernel's explicit wait for PV_{j-2} before it reuses a
    shared-memory P buffer never matters: one thread's MMAs complete in
    order, so the S_j commit that starts tile j already follows PV_{j-2};
    dropping the wait leaves every schedule clean."""
    for seed in range(300):
        m = Model("verify", 6, 2, 2, 3, rng=random.Random(seed), skip={"p_buffer"})
        m.run()
        assert not m.violations, m.violations[:3]


class DecodeRing:
    """The split-K decode kernels' ring (k_decode_split, k_decode_split_q8):
    one producer warp copies sub-block t into slot t % NSLOT after the slot's
    empty barrier says sub-block t - NSLOT was consumed; consumer warp w
    takes sub-blocks w, w + NCW, ...: it waits on the slot's full barrier,
    reads the slot and arrives on its empty barrier."""

    def __init__(self, n_sub, NSLOT, NCW, rng):
        self.n, self.NS, self.NCW, self.rng = n_sub, NSLOT, NCW, rng
        self.full = [Bar("full%d" % s, 1) for s in range(NSLOT)]
        self.empty = [Bar("empty%d" % s, 1) for s in range(NSLOT)]
        self.content = [None] * NSLOT   # sub-block whose rows a slot holds
        self.reading = [None] * NSLOT   # sub-block a consumer is reading from a slot
        self.inflight = []              # (slot, sub-block)
        self.violations = []

    def check_wait(self, bar, k):
        ret = (bar.phase & 1) != (k & 1)
        if ret != (bar.phase > k):
            self.violations.append("%s: wait for phase %d at phase %d returns %s" % (bar.name, k, bar.phase, ret))
        return ret

    def producer(self):
        for t in range(self.n):
            s = t % self.NS
            if t >= self.NS:
                while not self.check_wait(self.empty[s], t // self.NS - 1):
                    yield
            if self.reading[s] is not None:
                self.violations.append("copy of %d into slot %d while %d is read" % (t, s, self.reading[s]))
            self.inflight.append((s, t))
            yield

    def consumer(self, w):
        for t in range(w, self.n, self.NCW):
            s = t % self.NS
            while not self.check_wait(self.full[s], t // self.NS):
                yield
            if self.content[s] != t or any(x == s for x, _ in self.inflight):
                self.violations.append("sub-block %d read from slot %d holding %s" % (t, s, self.content[s]))
            self.reading[s] = t
            yield
            self.reading[s] = None
            self.empty[s].arrive()
            yield

    def run(self, max_steps=100000):
        agents = {"producer": self.producer()}
        for w in range(self.NCW):
            agents["consumer%d" % w] = self.consumer(w)
        done = set()
        for _ in range(max_steps):
            choices = [a for a in agents if a not in done] + (["copy"] if self.inflight else [])
            if not choices:
                return
            pick = self.rng.choice(choices)
            if pick == "copy":
                s, t = self.inflight.pop(self.rng.randrange(len(self.inflight)))
                self.content[s] = t
                self.full[s].arrive()
            else:
                try:
                    next(agents[pick])
                except StopIteration:
                    done.add(pick)
        self.violations.append("deadlock: %s still running" % sorted(set(agents) - done))


@pytest.mark.parametrize("NSLOT,NCW", [(3, 3), (6, 3)])
def test_decode_ring_as_built_has_no_race(NSLOT, NCW):
    """The ring sizes the decode kernels use (3 slots at bf16, 6 at int8, with
    three consumer warps) under random schedules."""
    for seed in range(300):
        for n_sub in (1, 2, 5, 13, 40):
            m = DecodeRing(n_sub, NSLOT, NCW, random.Random(seed))
            m.run()
            assert not m.violations, "n_sub %d seed %d: %s" % (n_sub, seed, m.violations[:3])


def test_decode_ring_needs_one_consumer_per_slot():
    """Why the kernels assert NSLOT % NCW == 0: with 4 slots and 3 consumer
    warps a slot's successive fills go to different warps, and a warp's
    parity wait can return for the fill before its own."""
    found = []
    for seed in range(2000):
        m = DecodeRing(40, 4, 3, random.Random(seed))
        m.run()
        found += m.violations
        if found:
            break
    assert found, "no violating schedule found"


# --------------------------------------------------------------------------- abort paths
class NamedBar:
    """A CTA barrier (bar.red.or / bar.sync on one id, or __syncthreads): a
    generation completes when all `count` warps have arrived; a bar.red.or
    returns the OR of their predicates. Every warp must make the same kind of
    call in the same generation."""

    def __init__(self, name, count, violations):
        self.name, self.count, self.violations = name, count, violations
        self.gen, self.arrived, self.result = 0, [], {}

    def arrive(self, warp, kind, pred=False):
        self.arrived.append((warp, kind, bool(pred)))
        if len(self.arrived) == self.count:
            kinds = {k for _, k, _ in self.arrived}
            if len(kinds) > 1:
                self.violations.append("%s: warps met at different calls %s" % (self.name, sorted(kinds)))
            self.result[self.gen] = any(p for _, _, p in self.arrived)
            self.gen += 1
            self.arrived = []


class VerifyAbortModel:
    """k_verify_tc's roles with their failure paths, one agent per warp:
    warp 0 the producer, warp 1 the MMA issuer, warps 2..5 the softmax. Any
    bounded wait may give up (its deadline passes): it raises the CTA's abort
    flag and returns false; later bounded waits see the flag and return false
    too. The softmax warps take every decision that leads to a named barrier
    by a vote, so they stay together; at the end all six warps meet at
    __syncthreads, then the producer waits (bounded, flag ignored) for its
    copies still in flight, and TMEM is released."""

    def __init__(self, n_tiles, MT, NSTAGE, rng, p_fail, mutate=None):
        self.n, self.MT, self.NS, self.rng, self.p_fail = n_tiles, MT, NSTAGE, rng, p_fail
        self.mutate = mutate  # a planted protocol mistake, to show the checks catch it
        self.violations = []
        B = Bar
        self.q_full = B("q_full", 1)
        self.full = [B("full%d" % s, 1) for s in range(NSTAGE)]
        self.empty = [B("empty%d" % s, 1) for s in range(NSTAGE)]
        self.s_full = [B("s_full%d" % i, 1) for i in range(2)]
        self.o_done = [B("o_done%d" % i, 1) for i in range(2)]
        self.p_ready = [B("p_ready%d" % i, 4) for i in range(2)]  # 128 threads: 4 warp arrivals
        self.drain = B("drain", 1)
        self.bar1 = NamedBar("bar1", 4, self.violations)        # the softmax warps' barrier
        self.block = NamedBar("syncthreads", 6, self.violations)
        self.abort = False
        self.tc_queue, self.tma_inflight = [], []
        self.issued, self.consumed = [0] * NSTAGE, [0] * NSTAGE
        self.q_issued = self.q_consumed = False
        self.expire = set()         # agents whose blocked bounded wait the scheduler times out
        self.blocked = {}           # agent -> (kind "bounded" | "barrier", can it move now?)
        self.softmax_ok = {}

    # -------------------------------------------------------------- primitives
    def bwait(self, agent, bar, k, honour_abort=True):
        """mbar_wait_bounded_at: True when phase k completed; False once the
        deadline passes (abort raised) or, when honour_abort, the flag is up."""
        if honour_abort and self.p_fail and self.rng.random() < self.p_fail:
            # this wait's deadline passes early (as for a copy that never lands);
            # the teardown waits are for copies that were issued and do land
            self.abort = True
            return False
        while True:
            if agent in self.expire:
                self.expire.discard(agent)
                self.abort = True
                self.blocked.pop(agent, None)
                return False
            if honour_abort and self.abort:
                self.blocked.pop(agent, None)
                return False
            if (bar.phase & 1) != (k & 1):
                if bar.phase <= k:
                    self.violations.append("%s: wait for phase %d at phase %d returns early" % (bar.name, k, bar.phase))
                self.blocked.pop(agent, None)
                return True
            self.blocked[agent] = ("bounded", lambda: (bar.phase & 1) != (k & 1) or (honour_abort and self.abort))
            yield

    def meet(self, agent, nb, kind, pred=False):
        gen = nb.gen
        nb.arrive(agent, kind, pred)
        while nb.gen == gen:
            self.blocked[agent] = ("barrier", lambda: nb.gen != gen)
            yield
        self.blocked.pop(agent, None)
        return nb.result[gen]

    # -------------------------------------------------------------- roles
    def producer(self):
        a = "w0"
        self.tma_inflight.append(("Q", self.q_full))
        self.q_issued = True
        item, ok = 0, True
        for j in range(self.n + 1):
            for kind in (0, 1):
                if not ok or (kind == 0 and j == self.n) or (kind == 1 and j == 0):
                    continue
                for _ in range(self.MT):
                    s = item % self.NS
                    if item >= self.NS:
                        ok = yield from self.bwait(a, self.empty[s], item // self.NS - 1)
                        if not ok:
                            break
                    self.issued[s] += 1
                    self.tma_inflight.append((s, self.full[s]))
                    item += 1
                    yield
        yield from self.meet(a, self.block, "syncthreads")
        if self.abort and self.mutate != "no_teardown_wait":  # copies in flight must land first
            if self.q_issued and not self.q_consumed:
                yield from self.bwait(a, self.q_full, 0, honour_abort=False)
            for s in range(self.NS):
                if self.issued[s] > self.consumed[s]:
                    yield from self.bwait(a, self.full[s], self.issued[s] - 1, honour_abort=False)
        if self.tma_inflight:
            self.violations.append("CTA exits with copies in flight: %s" % [x[0] for x in self.tma_inflight])

    def issuer(self):
        a = "w1"
        ok = yield from self.bwait(a, self.q_full, 0)
        if ok:
            self.q_consumed = True
        item = 0
        for j in range(self.n + 1):
            if not ok:
                break
            if j < self.n:
                for _ in range(self.MT):
                    s = item % self.NS
                    ok = yield from self.bwait(a, self.full[s], item // self.NS)
                    if not ok:
                        break
                    self.consumed[s] += 1
                    self.tc_queue.append(("mma", [self.empty[s]]))
                    item += 1
                    yield
                if not ok:
                    break
                self.tc_queue.append(("commit", [self.s_full[j & 1]]))
                yield
            if j >= 1:
                t = j - 1
                ok = yield from self.bwait(a, self.p_ready[t & 1], t >> 1)
                if not ok:
                    break
                for _ in range(self.MT):
                    s = item % self.NS
                    ok = yield from self.bwait(a, self.full[s], item // self.NS)
                    if not ok:
                        break
                    self.consumed[s] += 1
                    self.tc_queue.append(("mma", [self.empty[s]]))
                    item += 1
                    yield
                if not ok:
                    break
                self.tc_queue.append(("commit", [self.o_done[t & 1]]))
        # no MMA may be in flight when TMEM is released
        if self.mutate != "no_drain":
            self.tc_queue.append(("commit", [self.drain]))
            yield from self.bwait(a, self.drain, 0, honour_abort=False)
        yield from self.meet(a, self.block, "syncthreads")
        if any(op[0] == "mma" for op in self.tc_queue):
            self.violations.append("TMEM released with an MMA in flight")

    def softmax(self, w):
        a = "w%d" % (w + 2)
        ok, bad, pv_seen = True, False, 0
        for j in range(self.n):
            if not bad:
                got = yield from self.bwait(a, self.s_full[j & 1], j >> 1)
                bad = not got
            if self.mutate == "break_alone" and bad:
                ok = False
                break
            if (yield from self.meet(a, self.bar1, "red.or", bad)):
                ok = False
                break
            if (yield from self.meet(a, self.bar1, "red.or", self.rng.random() < 0.3)):  # some logit grew
                yield from self.meet(a, self.bar1, "sync")
                moved = yield from self.meet(a, self.bar1, "red.or", self.rng.random() < 0.5)
                if moved and j >= 1 and pv_seen < j:
                    got = yield from self.bwait(a, self.o_done[(j - 1) & 1], (j - 1) >> 1)
                    if got:
                        pv_seen = j
                    else:
                        bad = True
            if not bad and j >= 2 and pv_seen < j - 1:
                got = yield from self.bwait(a, self.o_done[j & 1], (j - 2) >> 1)
                if got:
                    pv_seen = j - 1
                else:
                    bad = True
            if bad:
                continue  # no arrival: the issuer's bounded wait sees the abort
            self.p_ready[j & 1].arrive()
            yield
        fin = ok and not bad
        if fin:
            t = self.n - 1
            fin = yield from self.bwait(a, self.o_done[t & 1], t >> 1)
        ok = not (yield from self.meet(a, self.bar1, "red.or", not fin))
        if ok:
            yield from self.meet(a, self.bar1, "sync")
            yield from self.meet(a, self.bar1, "sync")
        self.softmax_ok[w] = ok
        yield from self.meet(a, self.block, "syncthreads")

    # -------------------------------------------------------------- scheduler
    def run(self, max_steps=200000):
        agents = {"w0": self.producer(), "w1": self.issuer()}
        for w in range(4):
            agents["w%d" % (w + 2)] = self.softmax(w)
        done = set()
        for _ in range(max_steps):
            live = [x for x in agents if x not in done]
            engines = (["tc"] if self.tc_queue else []) + (["tma"] if self.tma_inflight else [])
            if not live and not engines:
                break
            runnable = [x for x in live if x not in self.blocked or self.blocked[x][1]()]
            progress = runnable + engines
            if not progress:
                stuck = [x for x in live if self.blocked[x][0] == "bounded"]
                if not stuck:
                    self.violations.append("deadlock at named barriers: %s" % sorted(live))
                    return
                self.expire.add(self.rng.choice(stuck))  # its deadline passes
                progress = stuck
            elif self.rng.random() < 0.2:
                progress = progress + [x for x in live if x not in runnable]  # polls that find nothing
            pick = self.rng.choice(progress)
            if pick == "tc":
                op = self.tc_queue.pop(0)
                for bar in op[1]:
                    bar.arrive()
            elif pick == "tma":
                _, bar = self.tma_inflight.pop(self.rng.randrange(len(self.tma_inflight)))
                bar.arrive()
            else:
                try:
                    next(agents[pick])
                except StopIteration:
                    done.add(pick)
        else:
            self.violations.append("did not finish: %s" % sorted(set(agents) - done))
            return
        if len(set(self.softmax_ok.values())) > 1:
            self.violations.append("softmax warps disagree on success: %s" % self.softmax_ok)
        if not self.abort and not all(self.softmax_ok.values()):
            self.violations.append("a run without timeouts failed")


@pytest.mark.parametrize("p_fail", [0.0, 0.002, 0.02, 0.2])
def test_multi_token_abort_paths_terminate_together(p_fail):
    """With bounded waits giving up at random points (and, when nothing can
    move, the deadline of a blocked wait passing), every warp of a
    multi-token CTA reaches the end: the softmax warps agree on the outcome,
    no named barrier is left half-met, TMEM is released only after the MMAs
    drain, and no copy is still in flight when the CTA exits. Without
    timeouts every run succeeds."""
    for seed in range(200):
        for shape in ((1, 1, 2), (4, 2, 3), (7, 4, 5)):
            m = VerifyAbortModel(*shape, rng=random.Random(seed), p_fail=p_fail)
            m.run()
            assert not m.violations, "p_fail %g seed %d shape %s: %s" % (p_fail, seed, shape, m.violations[:3])


@pytest.mark.parametrize("mutate", ["break_alone", "no_teardown_wait", "no_drain"])
def test_multi_token_abort_checks_have_teeth(mutate):
    """A softmax warp that leaves on its own failure instead of voting, a
    producer that does not wait for its copies in flight, an issuer that
    does not drain its MMAs: each is caught under random failures."""
    for seed in range(400):
        m = VerifyAbortModel(6, 2, 3, rng=random.Random(seed), p_fail=0.05, mutate=mutate)
        m.run()
        if m.violations:
            return
    pytest.fail("planted mistake %s not caught" % mutate)
