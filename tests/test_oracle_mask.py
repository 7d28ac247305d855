"""Pins for the oracle's block masks and CSR lists (no GPU).

Counts are checked against closed forms computed here by a different route (interval
arithmetic per row, or pair-counting formulas), never against the oracle's own loops.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle.mask import (all_mask, anchor_set, csr_to_dense, dense_to_csr, two_stage_mask,
                         window_anchor_mask)
from synthetic import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_tiny_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "mask_tiny.json")))
    m = window_anchor_mask(g["n_pad"], g["n_valid"], g["block_size"], g["unit_tokens"],
                           g["radius"], g["num_anchors"], g["step"])
    assert m.astype(int).tolist() == g["dense"]
    rp, ci = dense_to_csr(m)
    assert rp.tolist() == g["row_ptr"] and ci.tolist() == g["col_idx"]


def _window_count_closed_form(n_pad, n_valid, bs, U, r, G, s):
    """Row-by-row interval count: key blocks covering units [lo(i)-r, hi(i)+r], plus anchors."""
    nb = n_pad // bs
    last_unit = (n_valid - 1) // U
    anchors = {(a * nb // G + s) % nb for a in range(G)}
    total = 0
    lengths = []
    for i in range(nb):
        if i * bs >= n_valid:
            lo = hi = last_unit
        else:
            lo, hi = i * bs // U, (min((i + 1) * bs, n_valid) - 1) // U
        u0, u1 = max(0, lo - r), min(last_unit, hi + r)
        j0 = u0 * U // bs                                  # block holding the first token of unit u0
        j1 = min(n_valid - 1, (u1 + 1) * U - 1) // bs      # block holding the last token of unit u1
        if u1 == last_unit:
            j1 = nb - 1                                    # trailing padding blocks sit in the last unit
        cnt = (j1 - j0 + 1) + sum(1 for a in anchors if not (j0 <= a <= j1))
        lengths.append(cnt)
        total += cnt
    return total, lengths


@pytest.mark.parametrize("step", [0, 1, 17, 49])
def test_frame_window_count_small(step):
    w = WORKLOADS["small"]
    m = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, w.frame_tokens, 1, 4, step)
    total, lengths = _window_count_closed_form(w.n_pad, w.n_valid, w.block_size,
                                               w.frame_tokens, 1, 4, step)
    assert int(m.sum()) == total
    assert m.sum(axis=1).tolist() == lengths
    if step == 0:
        assert total == 10375 and min(lengths) == 28 and max(lengths) == 53


def test_padding_only_blocks_take_the_last_real_unit():
    # Hand-worked: 256 slots in 64-token blocks, 150 real tokens, units of 64 tokens, radius 0,
    # no anchors.  Blocks 0, 1 and 2 hold units 0, 1 and 2 (block 2: tokens 128..149).  Block 3
    # holds only padding and takes the unit of the last real token, 149 // 64 = 2.  With
    # radius 0 a block attends the blocks of its own unit: {0}, {1}, {2, 3}, {2, 3}.
    m = window_anchor_mask(256, 150, 64, 64, 0, 0, 0)
    assert m.astype(int).tolist() == [[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 1], [0, 0, 1, 1]]


@pytest.mark.parametrize("n_pad,n_valid,bs,U,r,G,s", [
    (1024, 700, 64, 100, 0, 3, 123),      # five trailing padding-only blocks
    (8192, 5000, 128, 1560, 2, 1, 0),     # frame windows, 25 padding-only blocks
    (640, 64, 64, 64, 1, 10, 7),          # one real block, every other block padding only
])
def test_window_rows_with_padding_only_blocks(n_pad, n_valid, bs, U, r, G, s):
    m = window_anchor_mask(n_pad, n_valid, bs, U, r, G, s)
    total, lengths = _window_count_closed_form(n_pad, n_valid, bs, U, r, G, s)
    assert m.sum(axis=1).tolist() == lengths and int(m.sum()) == total


def _band_count(nb, r, anchors):
    band = nb * (2 * r + 1) - r * (r + 1)
    extra = sum(nb - (min(nb - 1, a + r) - max(0, a - r) + 1) for a in anchors)
    return band + extra


@pytest.mark.parametrize("name,r", [("large", 28), ("large", 60), ("large", 171),
                                    ("long", 23), ("long", 48), ("long", 130), ("long", 287)])
def test_band_counts_closed_form(name, r):
    w = WORKLOADS[name]
    m = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, w.block_size, r, 4, 0)
    assert int(m.sum()) == _band_count(w.nb, r, anchor_set(w.nb, 4, 0))


def test_band_densities_hit_targets():
    # The radii of the density sweeps land within half a percent of 10/20/50 and 5/10/25/50 %.
    for name, rs, targets in [("large", (28, 60, 171), (0.10, 0.20, 0.50)),
                              ("long", (23, 48, 130, 287), (0.05, 0.10, 0.25, 0.50))]:
        w = WORKLOADS[name]
        for r, t in zip(rs, targets):
            dens = _band_count(w.nb, r, anchor_set(w.nb, 4, 0)) / w.nb**2
            assert abs(dens - t) < 0.005


def test_two_stage_closed_form():
    w = WORKLOADS["long"]
    g = int(round(math.sqrt(w.n_pad) / w.block_size))
    assert g == 3
    m = two_stage_mask(w.nb, g)
    full, rem = divmod(w.nb, g)
    local = full * g * g + rem * rem
    assert int(m.sum()) == local + w.nb == 3950       # strided block never falls in the own group
    for i in (0, 5, w.nb - 1):
        assert m[i, (i + g) % w.nb]


def test_rotation_covers_each_block_once():
    # LVSA: over T_per consecutive steps every frame is a global anchor exactly once.
    for nb, G in [(256, 4), (12, 3), (988, 4)]:
        if nb % G:
            continue
        t_per = nb // G
        seen = np.zeros(nb, dtype=int)
        for s in range(t_per):
            for a in anchor_set(nb, G, s):
                seen[a] += 1
        assert np.all(seen == 1)


def test_diagonal_always_active_and_all_mask():
    for r in (0, 1, 3):
        m = window_anchor_mask(1000, 977, 64, 100, r, 0, 0)
        assert np.all(np.diag(m))
    assert all_mask(7).sum() == 49


def test_frame_window_linear_in_frames():
    # LVSA complexity: with a fixed window the attended pairs grow linearly in T.
    # Frames of exactly 2 blocks, no anchors: second differences vanish once T > 2r+1.
    bs, U, r = 64, 128, 2
    counts = []
    for T in range(6, 12):
        n = T * U
        counts.append(int(window_anchor_mask(n, n, bs, U, r, 0, 0).sum()))
    d2 = np.diff(counts, 2)
    assert np.all(d2 == 0) and counts[1] - counts[0] == 4 * (2 * r + 1)


def test_csr_roundtrip_and_order():
    rng = np.random.default_rng(3)
    m = rng.random((3, 9, 9)) < 0.3
    m[1, 4] = False                                       # an empty row
    rp, ci = dense_to_csr(m)
    assert rp[0] == 0 and np.all(np.diff(rp) >= 0) and rp[-1] == m.sum()
    for row in range(27):
        seg = ci[rp[row]:rp[row + 1]]
        assert np.all(np.diff(seg) > 0)
    assert np.array_equal(csr_to_dense(rp, ci, 3, 9), m)


# ---------------------------------------------------------------- expanded LVSA windows
from oracle.mask import lvsa_frame_mask, lvsa_frame_sets  # noqa: E402


def test_lvsa_hand_worked_windows():
    g = json.load(open(os.path.join(GOLDEN, "lvsa_frames_hand.json")))
    for c in g["cases"]:
        anchors, windows, sets = lvsa_frame_sets(c["T"], c["G"], c["step"], c["C"])
        assert sorted(anchors) == c["anchors"]
        assert [list(w) for w in windows] == c["windows"], c["why"]


@pytest.mark.parametrize("T,G,C", [(21, 4, 21), (81, 4, 21), (126, 6, 21), (10, 3, 4), (5, 2, 9), (30, 0, 7)])
def test_lvsa_budget_invariant(T, G, C):
    # LVSA: the window is extended where it overlaps global frames so that |A(t)| = C
    # (or every frame when C >= T), at every step; W(t) is a contiguous interval holding t.
    for s in (0, 1, 7):
        anchors, windows, sets = lvsa_frame_sets(T, G, s, C)
        assert len(anchors) == min(G, T)
        for t, (lo, hi) in enumerate(windows):
            assert lo <= t <= hi
            assert sets[t] == anchors | set(range(lo, hi + 1))
            assert len(sets[t]) == min(C, T)


def test_lvsa_without_anchors_is_the_symmetric_window_inside():
    # G = 0, C = 2r + 1: interior frames get exactly [t - r, t + r].
    T, r = 40, 3
    _, windows, _ = lvsa_frame_sets(T, 0, 0, 2 * r + 1)
    for t in range(r, T - r):
        assert windows[t] == (t - r, t + r)
    assert windows[0] == (0, 2 * r) and windows[T - 1] == (T - 1 - 2 * r, T - 1)   # shifted inward


def test_lvsa_pairs_linear_in_frames():
    # Fixed budget: frame pairs = T * min(C, T), linear in T (LVSA complexity statement).
    for T in (30, 60, 120):
        _, _, sets = lvsa_frame_sets(T, 4, 0, 21)
        assert sum(len(a) for a in sets) == 21 * T


def test_lvsa_block_mask_from_frames():
    # Blocks aligned to frames (2 blocks per frame): block-level mask = frame-level sets expanded.
    T, fb, bs = 12, 2, 64
    U = fb * bs
    n = T * U
    m = lvsa_frame_mask(n, n, bs, U, 3, 2, 5)
    _, _, sets = lvsa_frame_sets(T, 3, 2, 5)
    for i in range(T * fb):
        for j in range(T * fb):
            assert m[i, j] == ((j // fb) in sets[i // fb])


def _cyclic_gaps(points, n):
    p = sorted(points)
    return [(p[(k + 1) % len(p)] - p[k]) % n or n for k in range(len(p))]


@pytest.mark.parametrize("n,G", [(10, 4), (21, 4), (81, 4), (591, 4), (988, 6), (7, 7), (13, 5)])
def test_anchors_spread_evenly_and_rotate(n, G):
    """Both anchor sets -- key blocks (window kind) and global frames (LVSA frames kind) --
    are G distinct positions spread as evenly as the count allows (cyclic gaps differ by at
    most one, LVSA page section 2: anchors spread over the sequence), and the step s shifts
    every one of them by s (the rotation of the global set)."""
    for s in (0, 1, 3, n - 1):
        block_anchors = anchor_set(n, G, s)
        frame_anchors, _, _ = lvsa_frame_sets(n, G, s, 1)
        for anchors in (block_anchors, frame_anchors):
            assert len(anchors) == G
            gaps = _cyclic_gaps(anchors, n)
            assert max(gaps) - min(gaps) <= 1, (n, G, s, sorted(anchors))
            assert anchors == {(a + s) % n for a in (anchor_set(n, G, 0) if anchors is block_anchors
                                                     else lvsa_frame_sets(n, G, 0, 1)[0])}
