"""Executable model of the block-energy kernel's mbarrier protocol (no GPU).

``block_energy_kernel`` (csrc/energy.cu) computes one energy row per CTA with three kinds
of roles:

* the TMA producer (warp 0): Q once, then K tiles into a 2-slot ring;
* the MMA issuer (warp 1): S_b = Q K^T into TMEM buffer b = t mod 2;
* the reduction warps (2..9): each reads its rows of S_b, sums its probabilities, and
  stores the warp sum for list position t in a shared [chunk x warps] buffer.  Every
  ``chunk`` positions (and at the end) the warps meet at a group barrier, each combines
  the eight warp sums of its share of the buffered positions in warp order and stores the
  energies, and they meet again before the buffer is reused.  The energy row is zeroed
  first, behind one more group barrier.  The group barrier is a pair of 8-count mbarriers
  used alternately: sync number q uses slot q mod 2 and waits for that slot's phase q div 2.

Built on ``tests.protocol_model`` (TMA copies land in any order, MMAs complete in issue
order; checks for deadlock, parity aliasing and buffer hazards).  In addition every
listed block's energy must end as the sum written after the row was zeroed.  The model
uses a chunk of 2 or 3 positions instead of 256 so that the chunk hand-off runs often;
the protocol does not depend on its size.
"""
import random

import pytest

from tests.protocol_model import Hazard, ProtocolModel

KST = 2              # K ring slots
WARPS = 3            # reduction warps modelled (8 in the kernel)


class EnergyModel(ProtocolModel):
    issuers = ("qk",)

    def __init__(self, n, nb, chunk, rng, omit=()):
        super().__init__(rng, omit)
        self.n, self.nb, self.chunk = n, nb, chunk
        self.cols = sorted(rng.sample(range(nb), n))           # the CSR row: n listed key blocks
        self.barrier("q", 1)
        self.barrier("final", 1)
        for s in range(KST):
            self.barrier(f"k_full{s}", 1)
            self.barrier(f"k_empty{s}", 1)
        for b in range(2):
            self.barrier(f"s_full{b}", 1)
            self.barrier(f"s_free{b}", WARPS)
            self.barrier(f"group{b}", WARPS)
        self.buffer("Q")
        for s in range(KST):
            self.buffer(f"K{s}")
        for w in range(WARPS):
            for b in range(2):
                self.buffer(f"S{b}w{w}")
        for x in range(chunk):
            for w in range(WARPS):
                self.buffer(f"R{x}w{w}")
        for j in range(nb):
            self.buffer(f"E{j}")

    def roles(self):
        return [self.producer(), self.issuer()] + [self.reducer(w) for w in range(WARPS)]

    def producer(self):
        if self.n == 0:
            return
        self.tma("Q", "q", "q")
        for t in range(self.n):
            s = t % KST
            if t >= KST:
                yield from self.wait(f"k_empty{s}", t // KST - 1, "k_empty")
            self.tma(f"K{s}", ("k", t), f"k_full{s}")
            yield

    def issuer(self):
        if self.n == 0:
            return
        yield from self.wait("q", 0, "q_full")
        for t in range(self.n):
            s, b = t % KST, t & 1
            yield from self.wait(f"k_full{s}", t // KST, "k_full")
            if t >= 2:
                yield from self.wait(f"s_free{b}", (t >> 1) - 1, "s_free")
            self.issue_mma("qk", [("Q", "q"), (f"K{s}", ("k", t))],
                           [(f"S{b}w{w}", ("s", t), None) for w in range(WARPS)])
            self.commit("qk", f"s_full{b}")
            self.commit("qk", f"k_empty{s}")
            yield
        self.commit("qk", "final")
        yield from self.wait("final", 0, "final")

    def reducer(self, w):
        seq = 0

        def group_sync(tag):
            nonlocal seq
            slot, phase = seq & 1, seq >> 1
            seq += 1
            self.bar[f"group{slot}"].arrive()
            yield from self.wait(f"group{slot}", phase, tag)

        for j in range(w, self.nb, WARPS):                  # the row starts at zero
            self.buf[f"E{j}"].write("zero", f"red{w}")
            yield
        yield from group_sync("zeroed")
        flushed = 0
        for t in range(self.n):
            b = t & 1
            yield from self.wait(f"s_full{b}", t >> 1, "s_full")
            self.buf[f"S{b}w{w}"].begin_read(("s", t))
            yield                                           # tcgen05.ld of the S rows
            self.buf[f"S{b}w{w}"].end_read()
            self.bar[f"s_free{b}"].arrive()
            self.buf[f"R{t - flushed}w{w}"].write(("r", t), f"red{w}")
            yield
            if t - flushed == self.chunk - 1 or t == self.n - 1:
                yield from group_sync("sums_stored")        # every warp sum of the chunk is stored
                for x in range(w, t - flushed + 1, WARPS):  # this warp's share of the positions
                    for v in range(WARPS):
                        self.buf[f"R{x}w{v}"].begin_read(("r", flushed + x))
                    yield                                   # add the warp sums in warp order
                    for v in range(WARPS):
                        self.buf[f"R{x}w{v}"].end_read()
                    self.buf[f"E{self.cols[flushed + x]}"].write(("e", flushed + x), f"red{w}")
                yield from group_sync("sums_read")          # the buffer may be refilled
                flushed = t + 1

    def finished(self):
        for t, j in enumerate(self.cols):
            if self.buf[f"E{j}"].version != ("e", t):
                raise Hazard(f"energy of block {j} ends as {self.buf[f'E{j}'].version}")
        for j in set(range(self.nb)) - set(self.cols):
            if self.buf[f"E{j}"].version != "zero":
                raise Hazard(f"unlisted block {j} ends as {self.buf[f'E{j}'].version}")


def _run(n, chunk, seed, omit=()):
    rng = random.Random(seed)
    EnergyModel(n, max(n, 7), chunk, rng, omit).run()


@pytest.mark.parametrize("chunk", [2, 3])
def test_random_rows_and_schedules(chunk):
    for n in (0, 1, 2, 3, 4, 5, 7):
        for sched in range(60):
            _run(n, chunk, seed=1000 * n + sched)


# Each of these waits is needed on the normal path: without it (in the model only) some
# schedule breaks a check.
WAITS = ["k_empty", "q_full", "k_full", "s_free", "s_full", "sums_stored", "sums_read"]


@pytest.mark.parametrize("omit", WAITS)
def test_every_wait_is_needed(omit):
    caught = 0
    for sched in range(400):
        try:
            _run(7, 2, seed=sched, omit=(omit,))
        except Hazard:
            caught += 1
            if caught >= 3:
                break
    assert caught > 0, f"no schedule needs the {omit} wait"


@pytest.mark.parametrize("omit", ["zeroed", "final"])
def test_waits_implied_on_the_normal_path(omit):
    """Two waits are implied by others when no wait times out:

    * the group sync after zeroing the row, by the first ``sums_stored`` sync: every warp
      zeroes its share before it arrives there, and energies are stored only after it;
    * the issuer's final drain, by the reduction warps' s_full waits: every MMA has
      completed before they finish and the CTA frees TMEM.

    The kernel keeps both: the first as an explicit ordering of the zero stores, the drain
    for the abort path.  Without them no schedule breaks a check."""
    for n in (0, 1, 5):
        for sched in range(150):
            _run(n, 2, seed=sched, omit=(omit,))
