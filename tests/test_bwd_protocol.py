"""A model of the backward kernel's hand-off protocol (csrc/attn_bwd.cu, one CTA), run under random
timings on the CPU.

The roles are coroutines: the TMA producer, the MMA issuer (its products run in issue order on an
asynchronous tensor pipe, and a commit arrives once every product issued before it is done), the
elementwise warps, the dQ warps and the end-of-unit dK/dV store. Every tensor-memory column range
and shared-memory buffer holds a tagged version ("S 3" = S^T of step 3). The checks:

- every wait on an mbarrier targets one phase and sees it complete without the barrier having moved
  two phases past it (a parity wait cannot tell those apart);
- every read finds the version it expects, and nothing is written while it is being read;
- all roles finish (no wait is left without its arrival).

The model follows the kernel's order of waits, arrivals, commits and accesses step by step; its
durations are random and roles are now and then held up for long stretches, so each seed is another
interleaving. Two tests plant mistakes in the model (not in the kernel) to show the checks bite: dQ's
columns released before they are read, and one barrier instead of two alternating slots for dK's
completion (caught as parity aliasing in some interleavings).
"""
import heapq
import random

import pytest


class Hazard(AssertionError):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phases = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phases += 1
            return True
        return False


class Resource:
    def __init__(self, name):
        self.name, self.version, self.readers, self.writer = name, None, 0, None


class Sim:
    def __init__(self, seed, stall_p=0.03, stall_max=60.0):
        self.rng = random.Random(seed)
        self.stall_p, self.stall_max = stall_p, stall_max
        self.now = 0.0
        self.queue = []  # (time, order, callback)
        self.order = 0
        self.bars = {}
        self.res = {}
        self.waiting = []  # (barrier, phase, resume)
        self.pipe_free_at = 0.0
        self.commits = []  # (products issued before the commit, barrier)
        self.pipe_done = 0
        self.pipe_issued = 0
        self.finished = set()

    # -- infrastructure ---------------------------------------------------------------------------
    def at(self, t, fn):
        self.order += 1
        heapq.heappush(self.queue, (t, self.order, fn))

    def jitter(self, base):
        return base * (0.5 + self.rng.random())

    def bar(self, name, count=1):
        self.bars[name] = Barrier(name, count)

    def r(self, name):
        if name not in self.res:
            self.res[name] = Resource(name)
        return self.res[name]

    def arrive(self, name):
        b = self.bars[name]
        if b.arrive():
            still = []
            for (bb, ph, resume) in self.waiting:
                if bb is b:
                    self.check_phase(bb, ph)
                    if bb.phases >= ph + 1:
                        self.at(self.now, resume)
                        continue
                still.append((bb, ph, resume))
            self.waiting = still

    def check_phase(self, b, ph):
        if b.phases > ph + 1:
            raise Hazard(f"{b.name}: waited for phase {ph} but {b.phases} phases had completed (parity aliasing)")

    def read_begin(self, name, expect):
        res = self.r(name)
        if res.writer is not None:
            raise Hazard(f"{name}: read of '{expect}' while '{res.writer}' is being written")
        if res.version != expect:
            raise Hazard(f"{name}: read expected '{expect}', found '{res.version}'")
        res.readers += 1

    def read_end(self, name):
        self.r(name).readers -= 1

    def write_begin(self, name, tag):
        res = self.r(name)
        if res.readers:
            raise Hazard(f"{name}: '{tag}' written while '{res.version}' is being read")
        if res.writer is not None:
            raise Hazard(f"{name}: '{tag}' written while '{res.writer}' is being written")
        res.writer = tag

    def write_end(self, name):
        res = self.r(name)
        res.version, res.writer = res.writer, None

    # -- role commands (generators yield these) ----------------------------------------------------
    def run(self, name, gen):
        def step(value=None):
            try:
                cmd = gen.send(value)
            except StopIteration:
                self.finished.add(name)
                return
            # now and then a role is held up for a long while before its next command (a warp not
            # scheduled), so that orderings which need one role to fall far behind occur too
            if self.rng.random() < self.stall_p:
                self.at(self.now + self.rng.uniform(0.0, self.stall_max), lambda: do(cmd))
            else:
                do(cmd)

        def do(cmd):
            kind = cmd[0]
            if kind == "delay":
                self.at(self.now + self.jitter(cmd[1]), step)
            elif kind == "wait":
                b, ph = self.bars[cmd[1]], cmd[2]
                self.check_phase(b, ph)
                if b.phases >= ph + 1:
                    self.at(self.now + self.jitter(1.0), step)
                else:
                    self.waiting.append((b, ph, step))
            elif kind == "arrive":
                self.arrive(cmd[1])
                self.at(self.now, step)
            elif kind == "access":  # synchronous: reads and writes held for a duration
                _, reads, writes, dur = cmd
                for (n, v) in reads:
                    self.read_begin(n, v)
                for (n, v) in writes:
                    self.write_begin(n, v)

                def done():
                    for (n, _) in reads:
                        self.read_end(n)
                    for (n, _) in writes:
                        self.write_end(n)
                    step()
                self.at(self.now + self.jitter(dur), done)
            elif kind == "async":  # a copy or a product off the role's thread: returns at once
                _, reads, writes, dur, on_done = cmd
                self.async_op(reads, writes, dur, on_done)
                self.at(self.now, step)
            elif kind == "mma":
                _, reads, writes = cmd
                self.issue_mma(reads, writes)
                self.at(self.now, step)
            elif kind == "commit":
                self.commits.append((self.pipe_issued, cmd[1]))
                self.check_commits()
                self.at(self.now, step)
            else:
                raise ValueError(kind)
        self.at(self.now, step)

    def async_op(self, reads, writes, dur, on_done):
        def begin():
            for (n, v) in reads:
                self.read_begin(n, v)
            for (n, v) in writes:
                self.write_begin(n, v)
            self.at(self.now + self.jitter(dur), end)

        def end():
            for (n, _) in reads:
                self.read_end(n)
            for (n, _) in writes:
                self.write_end(n)
            if on_done:
                on_done()
        self.at(self.now + self.jitter(0.5), begin)

    def issue_mma(self, reads, writes):
        self.pipe_issued += 1
        start = max(self.now + self.jitter(0.3), self.pipe_free_at)
        dur = self.jitter(4.0)
        self.pipe_free_at = start + dur

        written = {n for (n, _) in writes}
        plain_reads = [(n, v) for (n, v) in reads if n not in written]
        accumulated = [(n, v) for (n, v) in reads if n in written]  # read-modify-write by this product

        def begin():
            for (n, v) in plain_reads:
                self.read_begin(n, v)
            for (n, v) in accumulated:
                if self.r(n).version != v or self.r(n).writer is not None:
                    raise Hazard(f"{n}: accumulation expected '{v}', found '{self.r(n).version}'")
            for (n, v) in writes:
                self.write_begin(n, v)

        def end():
            for (n, _) in plain_reads:
                self.read_end(n)
            for (n, _) in writes:
                self.write_end(n)
            self.pipe_done += 1
            self.check_commits()
        self.at(start, begin)
        self.at(start + dur, end)

    def check_commits(self):
        ready = [c for c in self.commits if c[0] <= self.pipe_done]
        self.commits = [c for c in self.commits if c[0] > self.pipe_done]
        for (_, name) in ready:
            self.arrive(name)

    def go(self, limit=1e7):
        while self.queue:
            t, _, fn = heapq.heappop(self.queue)
            if t > limit:
                break
            self.now = t
            fn()


BARRIERS = ("kv_full", "q_full0", "q_full1", "q_empty0", "q_empty1", "st_full", "s_full", "pt_full", "p_full",
            "dq_full", "dq_free", "dk_done0", "dk_done1", "dkv_full", "epi_full", "epi_free")
ROLES = {"producer", "mma", "elementwise", "store", "dq"}


def backward_cta(sim, n_steps, early_release=False, single_dk=False):
    """Starts the roles of one backward CTA over n_steps steps (one key block). Each barrier takes one
    arrival per phase here (the kernel's counts are per warp; a role stands for its warps).

    early_release and single_dk plant mistakes (for the tests that show the model can catch them):
    the dQ warps release dQ's columns before reading them out, or dK's completion is tracked in one
    barrier for every step instead of two slots used on alternate steps."""
    for name in BARRIERS:
        sim.bar(name)
    if single_dk:
        sim.bars["dk_done1"] = sim.bars["dk_done0"]

    def producer():
        yield ("async", [], [("K", "K"), ("V", "V")], 6.0, lambda: sim.arrive("kv_full"))
        for t in range(n_steps):
            st = t & 1
            if t >= 2:
                yield ("wait", f"q_empty{st}", (t - 2) >> 1)
            yield ("async", [], [(f"Q{st}", f"Q {t}"), (f"dO{st}", f"dO {t}"), (f"LD{st}", f"LD {t}")], 6.0,
                   (lambda s=st: sim.arrive(f"q_full{s}")))

    def mma():
        yield ("wait", "kv_full", 0)
        for t in range(n_steps):
            st = t & 1
            yield ("wait", f"q_full{st}", t >> 1)
            if t > 0:
                yield ("wait", "dq_free", t - 1)                 # dQ of the last step read out
            yield ("mma", [("K", "K"), (f"Q{st}", f"Q {t}")], [("S", f"S {t}")])
            yield ("commit", "st_full")
            yield ("mma", [("V", "V"), (f"dO{st}", f"dO {t}")], [("DP", f"DP {t}")])
            yield ("commit", "s_full")
            yield ("wait", "pt_full", t)
            acc = [("DV", "DV")] if t > 0 else []
            yield ("mma", [("S", f"P {t}"), (f"dO{st}", f"dO {t}")] + acc, [("DV", "DV")])
            yield ("wait", "p_full", t)
            yield ("mma", [("dS", f"dS {t}"), ("K", "K")], [("S", f"dQ {t}")])
            yield ("commit", "dq_full")
            acc = [("DK", "DK")] if t > 0 else []
            yield ("mma", [("DP", f"dS^T {t}"), (f"Q{st}", f"Q {t}")] + acc, [("DK", "DK")])
            yield ("commit", f"dk_done{t & 1}")
            if t == n_steps - 1:
                yield ("commit", "dkv_full")

    def elementwise():
        for t in range(n_steps):
            st = t & 1
            yield ("wait", "st_full", t)
            yield ("access", [(f"LD{st}", f"LD {t}")], [], 1.0)
            yield ("access", [("S", f"S {t}")], [], 2.0)         # S^T read out
            yield ("delay", 6.0)                                 # exponentials
            yield ("access", [], [("S", f"P {t}")], 1.0)         # P^T over S^T
            yield ("arrive", "pt_full")
            yield ("wait", "s_full", t)
            yield ("access", [("DP", f"DP {t}"), (f"LD{st}", f"LD {t}")], [], 2.0)
            yield ("access", [], [("DP", f"dS^T {t}"), ("dS", f"dS {t}")], 2.0)
            yield ("arrive", "p_full")
        if n_steps == 0:
            return
        # end of the key block: dK and dV through the dS tile and TMA stores
        yield ("wait", "dkv_full", 0)
        for which, name in enumerate(("DK", "DV")):
            yield ("access", [(name, name)], [("dS", f"epi {name}")], 2.0)
            yield ("arrive", "epi_full")
            yield ("wait", "epi_free", which)

    def epilogue_store():
        if n_steps == 0:
            return
        for which, name in enumerate(("DK", "DV")):
            yield ("wait", "epi_full", which)
            done = []                                            # the store's read completion
            yield ("async", [("dS", f"epi {name}")], [], 3.0, lambda: done.append(1))
            while not done:
                yield ("delay", 0.5)
            yield ("arrive", "epi_free")

    def dq_warps():
        for t in range(n_steps):
            st = t & 1
            yield ("wait", "dq_full", t)
            if early_release:
                yield ("arrive", "dq_free")
                yield ("delay", 8.0)
            yield ("access", [("S", f"dQ {t}")], [(f"dO{st}", f"dQ hi {t}")], 2.0)  # columns 64..127
            reads = []
            yield ("async", [(f"dO{st}", f"dQ hi {t}")], [], 3.0, lambda: reads.append(1))
            yield ("access", [("S", f"dQ {t}")], [], 1.0)                            # columns 0..63
            if not early_release:
                yield ("arrive", "dq_free")
            if single_dk:
                yield ("wait", "dk_done0", t)
            else:
                yield ("wait", f"dk_done{t & 1}", t >> 1)
            yield ("access", [], [(f"Q{st}", f"dQ lo {t}")], 1.0)
            yield ("async", [(f"Q{st}", f"dQ lo {t}")], [], 3.0, lambda: reads.append(1))
            while len(reads) < 2:                                # both reduce-adds have read their boxes
                yield ("delay", 0.5)
            yield ("arrive", f"q_empty{st}")

    for name, gen in (("producer", producer()), ("mma", mma()), ("elementwise", elementwise()),
                      ("store", epilogue_store()), ("dq", dq_warps())):
        sim.run(name, gen)


@pytest.mark.parametrize("n_steps", [1, 2, 3, 7, 16])
def test_backward_protocol_has_no_hazard_and_finishes(n_steps):
    for seed in range(60):
        sim = Sim(1000 * n_steps + seed)
        backward_cta(sim, n_steps)
        sim.go()
        assert sim.finished == ROLES, f"seed {seed}: roles left waiting: {sorted(ROLES - sim.finished)}"
        assert sim.pipe_done == sim.pipe_issued == 5 * n_steps


def _caught(n_steps, seeds, **planted):
    caught = 0
    for seed in range(seeds):
        sim = Sim(seed)
        backward_cta(sim, n_steps, **planted)
        try:
            sim.go()
        except Hazard:
            caught += 1
            continue
        if sim.finished != ROLES:
            caught += 1
    return caught


def test_the_model_catches_a_release_before_the_read():
    """Planted mistake (in the model): dQ's columns released before they are read out; the next
    step's S^T may then overwrite dQ first."""
    assert _caught(4, 40, early_release=True) > 0


def test_the_model_catches_a_single_dk_barrier():
    """Planted mistake (in the model): one dk_done barrier for every step. With the columns released
    before that wait, the next step's dK can complete too before the dQ warps look, and a parity
    wait cannot tell the two phases apart."""
    assert _caught(8, 300, single_dk=True) > 0
