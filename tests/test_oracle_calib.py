"""Pins for the oracle's energy-based block selection and aggregation (no GPU).

Energies are checked against the attention matrix built by a library softmax and summed
by reshaping (another route), against closed forms (row sums, identical keys), and the
selection against hand-worked rows and an exhaustive subset search.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.calib import aggregate_masks, block_energy, select_blocks, select_row

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_qk(B, H, n_pad, n_valid, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, n_pad, d, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, H, n_pad, d, generator=g) * 1.5 + 0.3).to(torch.bfloat16)
    q[:, :, n_valid:] = 0
    k[:, :, n_valid:] = 0
    return q, k


@pytest.mark.parametrize("n_pad,n_valid,bs,d", [(128, 128, 32, 16), (192, 150, 64, 32), (256, 201, 64, 8)])
def test_energy_matches_library_softmax(n_pad, n_valid, bs, d):
    q, k = _rand_qk(2, 2, n_pad, n_valid, d, seed=n_valid)
    scale = 0.37
    e = block_energy(q, k, bs, n_valid, scale)
    nb = n_pad // bs
    qd, kd = q.double(), k.double()
    s = float(np.float32(scale)) * qd @ kd.transpose(-1, -2)          # [B,H,n_pad,n_pad]
    s[..., n_valid:] = float("-inf")
    a = torch.softmax(s, dim=-1)
    a[:, :, n_valid:, :] = 0.0                                         # padding rows carry no energy
    ref = a.reshape(2, 2, nb, bs, nb, bs).sum(dim=(3, 5)).numpy()
    np.testing.assert_allclose(e, ref, rtol=1e-12, atol=1e-12)


def test_energy_row_sums_count_real_rows():
    n_pad, n_valid, bs = 320, 250, 64
    q, k = _rand_qk(1, 3, n_pad, n_valid, 16, seed=7)
    e = block_energy(q, k, bs, n_valid, 0.5)
    rows = np.array([max(0, min((i + 1) * bs, n_valid) - i * bs) for i in range(n_pad // bs)], float)
    np.testing.assert_allclose(e.sum(axis=-1), np.broadcast_to(rows, e.shape[:-1]), rtol=1e-12)


def test_energy_identical_keys_is_uniform():
    # all keys equal: every real key gets probability 1/N, so E[i][j] = rows_i * keys_j / N
    n_pad, n_valid, bs, d = 256, 230, 64, 8
    q, _ = _rand_qk(1, 1, n_pad, n_valid, d, seed=3)
    k = torch.zeros(1, 1, n_pad, d, dtype=torch.bfloat16)
    k[:, :, :n_valid] = torch.linspace(-1, 1, d).to(torch.bfloat16)
    e = block_energy(q, k, bs, n_valid, 0.9)[0, 0]
    nb = n_pad // bs
    cnt = np.array([max(0, min((i + 1) * bs, n_valid) - i * bs) for i in range(nb)], float)
    np.testing.assert_allclose(e, np.outer(cnt, cnt) / n_valid, rtol=1e-12, atol=1e-15)


def test_energy_concentrates_on_the_matching_block():
    # one key per query row far more similar than the rest: energy sits on that key's block
    n_pad, bs, d = 256, 64, 32
    q = torch.zeros(1, 1, n_pad, d)
    k = torch.zeros(1, 1, n_pad, d)
    for r in range(n_pad):
        q[0, 0, r, r % d] = 8.0
    for c in range(n_pad):
        k[0, 0, c, (c * 5) % d] = 8.0 if c // bs == 2 else 0.0
    e = block_energy(q.to(torch.bfloat16), k.to(torch.bfloat16), bs, n_pad, 1.0)[0, 0]
    assert (e[:, 2] > 0.99 * bs).all()


def test_selection_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "energy_select_hand.json")))
    for case in g["select"]:
        got = select_row(np.array(case["energy"], dtype=np.float32), case["eps"])
        assert got.astype(int).tolist() == case["mask"], case["note"]
    masks = np.array(g["aggregate"]["masks"], dtype=np.uint8)
    for case in g["aggregate"]["cases"]:
        assert aggregate_masks(masks, case["rho"]).astype(int).tolist() == case["mask"], case["note"]


def test_selection_is_minimal_by_exhaustive_search():
    # small integer energies are exact in float64, so the threshold can be checked exactly
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 8))
        e = rng.integers(0, 6, size=n).astype(np.float32)
        eps = float(rng.choice([0.0, 0.25, 0.5, 0.6, 0.9, 1.0]))
        got = select_row(e, eps)
        total = int(e.sum())
        # the threshold is the float64 product eps * total (the reading); sums are exact here
        target = Fraction(float(eps) * float(total))
        best = None
        for kk in range(n + 1):
            if any(sum(Fraction(int(e[j])) for j in sub) >= target for sub in itertools.combinations(range(n), kk)):
                best = kk
                break
        assert int(got.sum()) == best, (e, eps, got)
        # the chosen blocks are a top-k set: nothing left out is larger than anything taken
        if got.any() and (~got).any():
            assert e[got].min() >= e[~got].max()
        # among equal energies at the cut, the lower indices are taken
        if got.any() and (~got).any():
            cut = e[got].min()
            taken = np.flatnonzero(got & (e == cut))
            left = np.flatnonzero(~got & (e == cut))
            if taken.size and left.size:
                assert taken.max() < left.min()


def test_select_blocks_rows_are_independent():
    rng = np.random.default_rng(5)
    e = rng.random((2, 3, 5, 7)).astype(np.float32)
    m = select_blocks(e, 0.7)
    for idx in np.ndindex(e.shape[:-1]):
        assert (m[idx] == select_row(e[idx], 0.7)).all()


def test_aggregate_extremes():
    rng = np.random.default_rng(9)
    masks = rng.random((5, 4, 6)) < 0.4
    assert (aggregate_masks(masks, 1.0) == masks.all(axis=0)).all()
    assert (aggregate_masks(masks, 0.2) == masks.any(axis=0)).all()
    assert aggregate_masks(masks, 0.0).all()
