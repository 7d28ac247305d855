"""Building blocks for CPU models of the kernels' mbarrier protocols (test helper).

A model replays each warp role of a kernel as a Python generator: its barrier waits (which
yield ``BLOCKED`` until the awaited phase completes), its arrivals, and its reads and writes
of shared-memory / TMEM buffers, in the kernel's order.  TMA copies land in any order;
each MMA issuer's MMAs complete in issue order, and a commit arrives once every MMA its
thread issued before it has completed.  A seeded random scheduler interleaves roles and
completions and raises ``Hazard`` on:

* deadlock (every live role waits and nothing is in flight) or no termination;
* phase aliasing: a wait for phase k begins with its barrier not at k or k + 1 completed
  phases, or ends at other than k + 1 (an mbarrier parity test cannot tell them apart);
* a buffer written while a read of it is in flight, or while another agent's write is in
  flight; a buffer read while a write is in flight or holding other content than expected;
* teardown (every role finished) with copies or MMAs still in flight.

Waits carry a tag; tags listed in ``omit`` are skipped, to show that a check catches the
absence of a wait (a mistake planted in the model only).
"""
import random

BLOCKED = "blocked"


class Hazard(AssertionError):
    pass


class Barrier:
    """An mbarrier: completed phases and the arrivals of the current phase."""

    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.completed = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived, self.completed = 0, self.completed + 1


class Buffer:
    """What a buffer holds, the reads of it in flight, and the writes to it in flight."""

    def __init__(self, name):
        self.name, self.version, self.reads, self.writes, self.writer = name, None, 0, 0, None

    def begin_write(self, version, writer, expect=None):
        if self.reads:
            raise Hazard(f"{self.name}: written ({version}) while {self.reads} read(s) of {self.version} in flight")
        if self.writes and self.writer != writer:
            raise Hazard(f"{self.name}: written by {writer} while a write by {self.writer} is in flight")
        if expect is not None and self.version != expect:
            raise Hazard(f"{self.name}: read-modify-write expects {expect}, holds {self.version}")
        self.version, self.writes, self.writer = version, self.writes + 1, writer

    def end_write(self):
        self.writes -= 1

    def write(self, version, writer):
        """A write that completes at once (plain stores by one thread)."""
        self.begin_write(version, writer)
        self.end_write()

    def begin_read(self, version):
        if self.writes:
            raise Hazard(f"{self.name}: read while a write ({self.version}) is in flight")
        if self.version != version:
            raise Hazard(f"{self.name}: read expects {version}, holds {self.version}")
        self.reads += 1

    def end_read(self):
        self.reads -= 1


class ProtocolModel:
    issuers = ()

    def __init__(self, rng, omit=()):
        self.rng, self.omit = rng, set(omit)
        self.bar, self.buf = {}, {}
        self.loads = []                                   # TMA copies in flight: (buffer, barrier)
        self.mma = {k: [] for k in self.issuers}          # per issuer, in issue order

    def barrier(self, name, count):
        self.bar[name] = Barrier(name, count)

    def buffer(self, name):
        self.buf[name] = Buffer(name)

    def wait(self, name, phase, tag):
        if tag in self.omit:
            return
        bar = self.bar[name]
        if not (phase <= bar.completed <= phase + 1):
            raise Hazard(f"{name}: wait for phase {phase} begins with {bar.completed} completed")
        while bar.completed == phase:
            yield BLOCKED
        if bar.completed != phase + 1:
            raise Hazard(f"{name}: wait for phase {phase} ends with {bar.completed} completed")

    def tma(self, buf, version, barrier):
        self.buf[buf].begin_write(version, "tma")
        self.loads.append((buf, barrier))

    def issue_mma(self, issuer, reads, writes):
        """reads: [(buffer, version)]; writes: [(buffer, new version, expected or None)]."""
        for name, version in reads:
            self.buf[name].begin_read(version)
        for name, version, expect in writes:
            self.buf[name].begin_write(version, issuer, expect)

        def complete():
            for name, _ in reads:
                self.buf[name].end_read()
            for name, _, _ in writes:
                self.buf[name].end_write()
        self.mma[issuer].append([complete])

    def commit(self, issuer, barrier):
        if self.mma[issuer]:
            self.mma[issuer][-1].append(lambda: self.bar[barrier].arrive())
        else:
            self.bar[barrier].arrive()

    def events(self):
        return [("load", i) for i in range(len(self.loads))] + [("mma", k) for k in self.issuers if self.mma[k]]

    def fire(self, ev):
        kind, x = ev
        if kind == "load":
            buf, barrier = self.loads.pop(x)
            self.buf[buf].end_write()
            self.bar[barrier].arrive()
        else:
            for f in self.mma[x].pop(0):
                f()

    def roles(self):
        raise NotImplementedError

    def run(self, max_steps=500000):
        live = list(self.roles())
        blocked = set()
        for _ in range(max_steps):
            evs = self.events()
            if not live and not evs:
                break
            kind, x = self.rng.choice([("role", r) for r in live] + [("ev", e) for e in evs])
            if kind == "ev":
                self.fire(x)
                blocked.clear()
                continue
            before = self._barrier_state()
            try:
                out = next(x)
            except StopIteration:
                live.remove(x)
                blocked.clear()
                if not live and evs:
                    raise Hazard(f"teardown with {len(self.loads)} load(s) and "
                                 f"{sum(map(len, self.mma.values()))} MMA(s) in flight")
                continue
            if out == BLOCKED and self._barrier_state() == before:
                # the role only re-checked its wait: nothing it did can release another role
                blocked.add(id(x))
                if not evs and all(id(r) in blocked for r in live):
                    raise Hazard("deadlock: every role waits and nothing is in flight")
            else:
                # it moved (an arrival, a copy or MMA issued, a buffer access): re-poll all
                blocked.clear()
                if out == BLOCKED:
                    blocked.add(id(x))
        else:
            raise Hazard("no termination")
        for name, b in self.buf.items():
            if b.reads or b.writes:
                raise Hazard(f"{name}: access in flight at exit")
        self.finished()

    def _barrier_state(self):
        return (tuple((b.completed, b.arrived) for b in self.bar.values()), len(self.loads),
                tuple(len(q) for q in self.mma.values()))

    def finished(self):
        """Checks on the final state (subclasses)."""


def random_decisions(rng, p):
    """A memoised coin per key: the same decision whenever a role asks again."""
    memo = {}

    def decide(*key):
        return memo.setdefault(key, rng.random() < p)
    return decide


__all__ = ["BLOCKED", "Hazard", "Barrier", "Buffer", "ProtocolModel", "random_decisions", "random"]
