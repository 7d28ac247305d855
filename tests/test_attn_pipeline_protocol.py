"""Executable model of the attention kernel's mbarrier protocol (no GPU).

``bsa_fwd_kernel`` (csrc/attn.cu) runs five kinds of roles that hand buffers to each other
through mbarriers whose waits test a phase *parity*:

* the Q/K producer (warp 0): Q once per item, then K tiles into a 3-slot ring;
* the V producer (warp 10): V tiles into a 3-slot ring;
* the Q K^T issuer (warp 1): S_b = Q K^T into TMEM buffer b = T mod 3, once O += P V of
  position T - 3 (which read P from that buffer) has completed;
* the P V issuer (warp 11): O += P_b V, with P_b read from TMEM over the first columns of S_b;
* the softmax warps (2..9), each owning rows of S, P and O: read S_b, write P_b over it,
  rescale O rarely, read O in the epilogue.  A key block after an item's first takes the
  speculative step: S_b read, and P_b written only once the block commits; a warp that
  gives the block up (its rows' max outgrew the reference) redoes it with the max-first
  step (S_b read again, P_b written, O rescaled), which is also the step of an item's first
  block.

The LSE-only form (``lva_block_sparse_lse``) runs the same roles without the V producer,
the P V issuer, P and O, with four S buffers: the softmax only reads S_b and releases it
(s_free), and the Q K^T issuer waits for that release.

Positions T count key blocks over all the items a CTA walks, so ring slots (T mod 3), S
buffers (T mod 3, or T mod 4) and barrier phases continue from one item to the next;
``q_empty`` and ``o_free`` hand the single Q tile and the O accumulator from one item to the
next.  Items with no key blocks (empty rows, corrupt rows, blocks skipped for repetitive
heads) take no part in the pipeline.

The model replays each role's waits, arrivals and buffer accesses in the kernel's order.
TMA loads land in any order; each issuer's MMAs complete in issue order, and a
``tcgen05.commit`` arrives once every MMA its thread issued before it has completed.  A
seeded random scheduler runs many item runs (empty items, rows of 1 to 5 key blocks, runs
of 1, 4 and 8 items, random redo and rescale decisions per warp) under many interleavings
and checks:

* progress: every run ends, with nothing in flight (no deadlock);
* no phase aliasing: a wait for phase k starts only when its barrier has completed k or
  k + 1 phases and ends at exactly k + 1 (a parity test cannot tell k from k + 2);
* no buffer hazard: a K/V ring slot, Q, or a warp's rows of S_b (or the P over it) or O are
  written only when no read of them is in flight (writes by one MMA issuer may overlap: its
  MMAs run in order), and read only once written, with the content the reader expects.
"""
import random

import pytest

from tests.protocol_model import Hazard, ProtocolModel, random_decisions

KST = VST = 3        # K and V ring slots
WARPS = 3            # softmax warps modelled (8 in the kernel; the protocol is per warp)


class Model(ProtocolModel):
    issuers = ("qk", "pv")

    def __init__(self, items, rescale, rng, omit=(), lse_only=False, redo=None, early_p=False):
        super().__init__(rng, omit)
        self.items, self.rescale, self.lse_only = items, rescale, lse_only
        self.redo = redo if redo is not None else (lambda *key: True)
        # a planted mistake: the speculative step releases S_b (LSE only) or writes P_b over
        # it (with P V) before it knows whether the block is redone
        self.early_p = early_p
        self.nsb = 4 if lse_only else 3
        for name, count in [("q", 1), ("q_empty", 1), ("o_free", WARPS), ("final", 1), ("final_pv", 1)]:
            self.barrier(name, count)
        for s in range(KST):
            self.barrier(f"k_full{s}", 1)
            self.barrier(f"k_empty{s}", 1)
        for s in range(VST):
            self.barrier(f"v_full{s}", 1)
            self.barrier(f"v_empty{s}", 1)
        for b in range(self.nsb):
            for name, count in [("s_full", 1), ("s_free", WARPS), ("p_full", WARPS), ("o_done", 1)]:
                self.barrier(f"{name}{b}", count)
        for name in ["Q"] + [f"K{s}" for s in range(KST)] + [f"V{s}" for s in range(VST)]:
            self.buffer(name)
        for w in range(WARPS):
            for b in range(self.nsb):
                self.buffer(f"S{b}w{w}")             # S_b, and P_b over its first columns
            self.buffer(f"Ow{w}")

    def roles(self):
        roles = [self.qk_producer(), self.qk_issuer()] + [self.softmax(w) for w in range(WARPS)]
        if not self.lse_only:
            roles += [self.v_producer(), self.pv_issuer()]
        return roles

    # -- the roles ----------------------------------------------------------------------------
    def qk_producer(self):
        T = nq = 0
        for it, n in enumerate(self.items):
            if n == 0:
                continue
            if nq > 0:
                yield from self.wait("q_empty", nq - 1, "q_empty")       # the previous item's Q K^T is done
            self.tma("Q", ("q", it), "q")
            nq += 1
            for _ in range(n):
                s = T % KST
                if T >= KST:
                    yield from self.wait(f"k_empty{s}", T // KST - 1, "k_empty")
                self.tma(f"K{s}", ("k", T), f"k_full{s}")
                T += 1
                yield

    def v_producer(self):
        T = 0
        for n in self.items:
            for _ in range(n):
                s = T % VST
                if T >= VST:
                    yield from self.wait(f"v_empty{s}", T // VST - 1, "v_empty")
                self.tma(f"V{s}", ("v", T), f"v_full{s}")
                T += 1
                yield

    def qk_issuer(self):
        T = nq = 0
        for it, n in enumerate(self.items):
            if n == 0:
                continue
            yield from self.wait("q", nq, "q_full")
            for _ in range(n):
                s, b = T % KST, T % self.nsb
                yield from self.wait(f"k_full{s}", T // KST, "k_full")
                if T >= self.nsb:
                    # S_b is free: released by the softmax (LSE only), or its P read by P V
                    free = f"s_free{b}" if self.lse_only else f"o_done{b}"
                    yield from self.wait(free, T // self.nsb - 1, "s_free")
                self.issue_mma("qk", [("Q", ("q", it)), (f"K{s}", ("k", T))],
                               [(f"S{b}w{w}", ("s", T), None) for w in range(WARPS)])
                self.commit("qk", f"s_full{b}")
                self.commit("qk", f"k_empty{s}")
                T += 1
                yield
            self.commit("qk", "q_empty")
            nq += 1
        self.commit("qk", "final")
        yield from self.wait("final", 0, "final")                     # drain before TMEM is released

    def pv_issuer(self):
        T = nq = 0
        for n in self.items:
            if n == 0:
                continue
            if nq > 0:
                yield from self.wait("o_free", nq - 1, "o_free")       # the previous item's O was read
            for t in range(n):
                s, b = T % VST, T % self.nsb
                yield from self.wait(f"p_full{b}", T // self.nsb, "p_full")
                yield from self.wait(f"v_full{s}", T // VST, "v_full")
                o_writes = [(f"Ow{w}", ("o", T), ("o", T - 1) if t > 0 else None) for w in range(WARPS)]
                self.issue_mma("pv", [(f"S{b}w{w}", ("p", T)) for w in range(WARPS)] + [(f"V{s}", ("v", T))],
                               o_writes)
                self.commit("pv", f"v_empty{s}")
                self.commit("pv", f"o_done{b}")
                T += 1
                yield
            nq += 1
        self.commit("pv", "final_pv")
        yield from self.wait("final_pv", 0, "final_pv")

    def softmax(self, w):
        T = 0
        nsb = self.nsb
        for it, n in enumerate(self.items):
            for t in range(n):
                b = T % nsb
                S = f"S{b}w{w}"
                if t >= 1:
                    # speculative step: P_b (over S_b) written only once the block commits
                    yield from self.wait(f"s_full{b}", T // nsb, "s_full")
                    self.buf[S].begin_read(("s", T))
                    yield                                    # tcgen05.ld of the S rows
                    self.buf[S].end_read()
                    if self.early_p:
                        if self.lse_only:
                            self.bar[f"s_free{b}"].arrive()
                        else:
                            self.buf[S].write(("p", T), f"sm{w}")
                    yield                                    # exponentials (and sums)
                    if not self.redo(w, it, t):
                        if self.lse_only:
                            if not self.early_p:
                                self.bar[f"s_free{b}"].arrive()
                        else:
                            if not self.early_p:
                                self.buf[S].begin_write(("p", T), f"sm{w}")
                                yield                        # tcgen05.st of P over S
                                self.buf[S].end_write()
                            self.bar[f"p_full{b}"].arrive()
                        T += 1
                        yield
                        continue
                # max-first step: an item's first block, or a block the warp gave up
                yield from self.wait(f"s_full{b}", T // nsb, "s_full")
                self.buf[S].begin_read(("s", T))
                yield                                        # tcgen05.ld of the S rows
                self.buf[S].end_read()
                if self.lse_only:
                    if not (self.early_p and t >= 1):
                        self.bar[f"s_free{b}"].arrive()
                    T += 1
                    yield                                    # maxima, exponentials, sums
                    continue
                self.buf[S].begin_write(("p", T), f"sm{w}")
                yield                                        # exponentials, tcgen05.st of P over S
                self.buf[S].end_write()
                if t >= 1 and self.rescale(w, it, t):
                    pb = (T - 1) % nsb
                    yield from self.wait(f"o_done{pb}", (T - 1) // nsb, "rescale")   # P V(T-1) is done
                    self.buf[f"Ow{w}"].begin_write(("o", T - 1), f"sm{w}", ("o", T - 1))
                    yield                                    # O rows scaled in TMEM
                    self.buf[f"Ow{w}"].end_write()
                self.bar[f"p_full{b}"].arrive()
                T += 1
                yield
            if n > 0 and not self.lse_only:
                yield from self.wait(f"o_done{(T - 1) % nsb}", (T - 1) // nsb, "epilogue")
                self.buf[f"Ow{w}"].begin_read(("o", T - 1))
                yield                                        # tcgen05.ld of the O rows
                self.buf[f"Ow{w}"].end_read()
                self.bar["o_free"].arrive()
            yield                                            # normalise, store O and LSE


def _run(items, seed, omit=(), lse_only=False):
    rng = random.Random(seed)
    Model(items, random_decisions(rng, 0.3), rng, omit, lse_only, redo=random_decisions(rng, 0.3)).run()


@pytest.mark.parametrize("lse_only", [False, True])
@pytest.mark.parametrize("kpc", [1, 4, 8])
def test_random_item_runs_and_schedules(kpc, lse_only):
    rng = random.Random(1000 + kpc)
    for case in range(40):
        items = [rng.choice([0, 0, 1, 1, 2, 3, 5]) for _ in range(kpc)]
        for sched in range(6):
            _run(items, seed=case * 100 + sched, lse_only=lse_only)


@pytest.mark.parametrize("items", [
    [1], [2], [5], [0], [0, 0, 0, 0],
    [1, 1, 1, 1, 1, 1, 1, 1],           # one key block per item: Q and O hand-offs at every block
    [0, 3, 0, 1, 0, 0, 2, 0],           # empty items between short rows
    [5, 0, 0, 0, 0, 0, 0, 1],
    [2, 2, 2, 2], [3, 1, 3, 1],         # positions cross ring and buffer boundaries inside items
])
def test_edge_item_runs(items):
    for sched in range(30):
        _run(items, seed=sched)
        _run(items, seed=sched, lse_only=True)


# Each of these waits is needed on the normal path: without it (in the model only) some
# schedule breaks a check.
WAITS = ["q_empty", "k_empty", "v_empty", "q_full", "k_full", "s_free", "p_full", "v_full",
         "s_full", "rescale", "epilogue"]


WAITS_LSE = ["q_empty", "k_empty", "q_full", "k_full", "s_free", "s_full"]


def _caught(omit, lse_only):
    caught = 0
    for sched in range(400):
        try:
            _run([5, 1, 3, 2], seed=sched, omit=(omit,), lse_only=lse_only)
        except Hazard:
            caught += 1
            if caught >= 3:
                break
    return caught


@pytest.mark.parametrize("omit", WAITS)
def test_every_wait_is_needed(omit):
    assert _caught(omit, False) > 0, f"no schedule needs the {omit} wait"


@pytest.mark.parametrize("omit", WAITS_LSE)
def test_every_wait_is_needed_lse_only(omit):
    assert _caught(omit, True) > 0, f"no schedule needs the {omit} wait (LSE only)"


@pytest.mark.parametrize("omit", ["o_free", "final", "final_pv"])
def test_waits_implied_on_the_normal_path(omit):
    """Three waits are implied by others when no wait times out:

    * o_free (an item's O read before the next item overwrites it) by p_full: a softmax
      warp arrives on p_full for the next item's first block only after its own epilogue
      has read O;
    * the issuers' final drains by the softmax: it waits for every S (s_full) and, in each
      epilogue, for the item's last P V (o_done), so every MMA has completed before the
      softmax warps finish and the CTA frees TMEM.

    The kernel keeps all three: o_free as an explicit hand-off, and the drains for the abort
    path, where the softmax warps may stop early.  Without them no schedule breaks a check."""
    for sched in range(200):
        _run([5, 1, 3, 2], seed=sched, omit=(omit,))
        _run([1, 1, 1, 1, 1, 1, 1, 1], seed=sched, omit=(omit,))


@pytest.mark.parametrize("lse_only", [False, True])
def test_speculative_step_must_hold_s_until_it_commits(lse_only):
    """A speculative step that released S_b (LSE only) or wrote P_b over it before knowing
    whether the block is redone would let a redo read something other than S: Q K^T(T+2)'s
    result, or P.  Some schedule shows the hazard.  The kernel writes P and releases S_b only
    once the block commits, or in the max-first step."""
    caught = 0
    for sched in range(600):
        rng = random.Random(sched)
        try:
            Model([5, 1, 3, 2], random_decisions(rng, 0.3), rng, lse_only=lse_only,
                  redo=random_decisions(rng, 0.5), early_p=True).run()
        except Hazard:
            caught += 1
            if caught >= 3:
                break
    assert caught > 0
