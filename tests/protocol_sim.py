"""A small discrete-event simulator for checking the kernels' hand-off protocols on the CPU.

Roles are Python generators that yield commands: wait for a given phase of an mbarrier, arrive on
one, access tagged resources for a while (reads expect a version, writes install one), start an
asynchronous copy, issue a tensor-core product (products run one after another in issue order) or
commit (arrive on a barrier once every product issued so far is done). Durations are random per
seed, and a role is now and then held up for a long stretch, so each seed is another interleaving.
Violations raise Hazard: a read that finds another version or overlaps a write, a write over a
resource being read, or a wait that finds its barrier two phases past the one it waits for (a parity
wait cannot tell those apart). A role left waiting when the events run out is a deadlock.
"""
import heapq
import random


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
