"""Pins for the oracle's tile permutation (no GPU)."""
import json
import os

import numpy as np
import pytest

from oracle.reorder import reorder_forward, reorder_inverse, tile_permutation
from synthetic import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_worked_permutations():
    cases = json.load(open(os.path.join(GOLDEN, "reorder_hand.json")))["cases"]
    for c in cases:
        perm = tile_permutation(c["T"], c["H"], c["W"], *c["tile"])
        assert perm.tolist() == c["perm"], c["why"]


@pytest.mark.parametrize("name", ["tiny", "small", "large", "long"])
def test_bijection(name):
    w = WORKLOADS[name]
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    assert perm.shape == (w.n_valid,)
    assert np.array_equal(np.sort(perm), np.arange(w.n_valid))


def _census(Hg, Wg, th, tw):
    """Closed form: tile sizes of one frame, in tile order, for tile depth 1."""
    hs = [th] * (Hg // th) + ([Hg % th] if Hg % th else [])
    ws = [tw] * (Wg // tw) + ([Wg % tw] if Wg % tw else [])
    return [a * b for a in hs for b in ws]


@pytest.mark.parametrize("name,expect", [
    ("small", {128: 9, 32: 3, 96: 3, 24: 1}),     # 30x52 grid, 8x16 tiles
    ("large", {128: 25, 80: 5}),                   # 45x80 grid, 8x16 tiles
])
def test_tile_census(name, expect):
    w = WORKLOADS[name]
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    sizes = _census(w.Hg, w.Wg, w.tile[1], w.tile[2])
    hist = {}
    for s in sizes:
        hist[s] = hist.get(s, 0) + 1
    assert hist == expect and sum(sizes) == w.frame_tokens
    # The permutation's runs of tokens sharing a tile id have exactly these sizes, frame by frame.
    t = perm // w.frame_tokens
    h = (perm // w.Wg) % w.Hg
    x = perm % w.Wg
    tid = (t // w.tile[0]) * 10**6 + (h // w.tile[1]) * 10**3 + (x // w.tile[2])
    change = np.flatnonzero(np.diff(tid)) + 1
    runs = np.diff(np.concatenate([[0], change, [perm.size]]))
    assert runs.tolist() == sizes * w.T


def test_roundtrip_and_padding():
    w = WORKLOADS["tiny"]
    rng = np.random.default_rng(5)
    perm = tile_permutation(3, 5, 7, 2, 2, 4)
    n = perm.size
    n_pad = 128
    src = rng.integers(-2**15, 2**15, size=(3, n, 4), dtype=np.int16)
    fwd = reorder_forward(src, perm, n_pad)
    assert np.all(fwd[:, n:] == 0)
    assert np.array_equal(reorder_inverse(fwd, perm), src)
    del w


def test_iota_returns_permutation():
    perm = tile_permutation(4, 6, 10, 1, 4, 8)
    iota = np.arange(perm.size, dtype=np.int32)[None, :, None]
    out = reorder_forward(iota, perm, perm.size + 16)
    assert np.array_equal(out[0, :perm.size, 0], perm)


def test_frames_stay_contiguous_with_unit_depth():
    # With tile depth 1 every frame's tokens occupy one contiguous range in tile order,
    # which is what lets a window measured in H*W-token units mean "latent frames".
    w = WORKLOADS["small"]
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    frames = perm // w.frame_tokens
    assert np.array_equal(frames, np.repeat(np.arange(w.T), w.frame_tokens))
