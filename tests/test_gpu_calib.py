"""Static-mask calibration through the C ABI vs the FP64 oracle: block energies (within a
tolerance), the threshold selection and the cross-prompt aggregation (bit-exact), and the
whole calibrator on several prompts."""
import numpy as np
import pytest
import torch

from oracle.calib import aggregate_masks, block_energy, select_blocks, select_row
from oracle.reorder import reorder_forward, tile_permutation
from synthetic import WORKLOADS, Workload, make_qk_calibration
from tests.gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu

# Energies: each probability is 2^(s*scale*log2e - LSE*log2e) with an fp32 score, the LSE of
# the attention call (|dLSE| well under 1e-4 on these inputs) and a 2^x of relative error
# <= 7.5e-5, summed in fp32 over <= 16384 terms: relative error <= ~3e-4 per block.
E_RTOL, E_ATOL = 2e-3, 1e-6

CASES = {
    "tiny": WORKLOADS["tiny"],
    # 600 tokens in 5 blocks of 128 (the last has 88 real rows and keys), B = 2
    "ragged": Workload("ragged", B=2, H=2, d=128, T=3, Hg=10, Wg=20, tile=(1, 5, 8), block_size=128, seed=21),
    "d64": Workload("d64", B=1, H=3, d=64, T=2, Hg=12, Wg=30, tile=(1, 4, 8), block_size=128, seed=22),
    "bs64": Workload("bs64", B=1, H=2, d=128, T=3, Hg=9, Wg=14, tile=(1, 3, 7), block_size=64, seed=23),
}


def _oracle_tile_order(w, x):
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    P = w.B * x.shape[1]
    out = reorder_forward(x.float().numpy().reshape(P, w.n_valid, w.d), perm, w.n_pad)
    return out.reshape(w.B, x.shape[1], w.n_pad, w.d)


def _gpu_energy(w, q, k, dev):
    import block_sparse_attention_lva_b200 as lva
    cal = lva.StaticMaskCalibrator(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size,
                                   scale=w.scale, device=dev)
    e = cal.energies(q.to(dev), k.to(dev)).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    return e


@pytest.mark.parametrize("name", list(CASES))
def test_energy_matches_oracle(name):
    dev = require_gpu()
    w = CASES[name]
    q, k = make_qk_calibration(w, prompt=0)
    got = _gpu_energy(w, q, k, dev)
    ref = block_energy(_oracle_tile_order(w, q), _oracle_tile_order(w, k), w.block_size, w.n_valid, w.scale)
    err = np.abs(got - ref)
    assert (err <= E_RTOL * ref + E_ATOL).all(), (err.max(), (err / (ref + 1e-30)).max())
    # every real query row carries probability 1 in total
    rows = np.array([max(0, min((i + 1) * w.block_size, w.n_valid) - i * w.block_size) for i in range(w.nb)])
    np.testing.assert_allclose(got.sum(axis=-1), np.broadcast_to(rows, got.shape[:-1]), rtol=1e-3, atol=1e-6)


def test_energy_full_size_sampled_rows():
    # 12 heads x 32,768 tokens; the oracle computes a few query blocks one by one, including
    # the block that holds the sequence end.
    dev = require_gpu()
    w = WORKLOADS["small"]
    q, k = make_qk_calibration(w, prompt=0)
    got = _gpu_energy(w, q, k, dev)
    samples = [(0, 0, 0), (0, 3, 17), (0, 7, 128), (0, 11, w.nb - 1), (0, 5, w.nb - 2)]
    heads = sorted({h for _, h, _ in samples})
    qt = _oracle_tile_order(w, q[:, heads])
    kt = _oracle_tile_order(w, k[:, heads])
    remap = {h: n for n, h in enumerate(heads)}
    ref = block_energy(qt, kt, w.block_size, w.n_valid, w.scale,
                       query_blocks=[(b, remap[h], i) for b, h, i in samples])
    for b, h, i in samples:
        r, g = ref[b, remap[h], i], got[b, h, i]
        assert (np.abs(g - r) <= E_RTOL * r + E_ATOL).all(), (h, i, np.abs(g - r).max())


def _energy_rows(rng, rows, nb):
    """Seeded energies with the features the selection must handle: heavy tails, exact ties
    (repeated values), zeros, and an all-zero row."""
    e = rng.exponential(1.0, size=(rows, nb)) ** 3
    e[rng.random((rows, nb)) < 0.2] = 0.0
    dup = rng.random((rows, nb)) < 0.3
    e[dup] = e[np.arange(rows)[:, None].repeat(nb, 1)[dup], rng.integers(0, nb, size=int(dup.sum()))]
    e[0] = 0.0
    return e.astype(np.float32)


@pytest.mark.parametrize("nb", [1, 3, 64, 256, 988, 4096])
def test_selection_bit_exact(nb):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    rng = np.random.default_rng(nb)
    rows = 6 if nb >= 988 else 40
    e = _energy_rows(rng, rows, nb)
    ed = torch.from_numpy(e).to(dev)
    for eps in (0.0, 0.3, 0.8, 0.95, 1.0):
        m = torch.empty((rows, nb), dtype=torch.uint8, device=dev)
        lva.lva_select_blocks(ed, m, eps)
        torch.cuda.synchronize()
        assert lva.lva_device_error() == (0, 0)
        assert np.array_equal(m.cpu().numpy().astype(bool), select_blocks(e, eps)), eps


def test_selection_rejects_invalid_energy_rows():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    e = np.abs(np.random.default_rng(3).normal(size=(4, 50))).astype(np.float32)
    e[2, 7] = -1.0
    m = torch.full((4, 50), 9, dtype=torch.uint8, device=dev)
    lva.lva_select_blocks(torch.from_numpy(e).to(dev), m, 0.9)
    st, detail = lva.lva_device_error()
    got = m.cpu().numpy()
    assert st == 1 and detail == 2
    assert (got[2] == 0).all()
    for r in (0, 1, 3):
        assert np.array_equal(got[r].astype(bool), select_row(e[r], 0.9))


@pytest.mark.parametrize("prompts", [1, 3, 8])
def test_aggregation_bit_exact(prompts):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    rng = np.random.default_rng(prompts)
    masks = (rng.random((prompts, 3, 37, 37)) < 0.45).astype(np.uint8)
    masks[masks == 1] = rng.integers(1, 255, size=int(masks.sum())).astype(np.uint8)   # any nonzero byte
    md = torch.from_numpy(masks).to(dev)
    for rho in (0.0, 0.25, 0.5, 2.0 / 3.0, 1.0):
        out = torch.empty((3, 37, 37), dtype=torch.uint8, device=dev)
        lva.lva_aggregate_masks(md, out, rho)
        assert np.array_equal(out.cpu().numpy().astype(bool), aggregate_masks(masks, rho)), rho


def test_calibrator_end_to_end():
    """Three prompts -> per-prompt selections -> aggregated static mask, against the oracle.
    A selection may differ only in a row whose cumulative energy sits within the energy
    tolerance of the threshold (then both counts are correct for some energy in range)."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    w = CASES["ragged"]
    eps, rho, n_prompts = 0.8, 0.5, 3
    cal = lva.StaticMaskCalibrator(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size,
                                   scale=w.scale, device=dev)
    ref_samples = []
    ambiguous = np.zeros((w.H, w.nb), dtype=bool)
    for p in range(n_prompts):
        q, k = make_qk_calibration(w, prompt=p)
        got = cal.add_prompt(q.to(dev), k.to(dev), eps).cpu().numpy().astype(bool)
        e_ref = block_energy(_oracle_tile_order(w, q), _oracle_tile_order(w, k), w.block_size, w.n_valid,
                             w.scale)
        ref = select_blocks(e_ref, eps)
        ref_samples.append(ref)
        for b, h, i in zip(*np.nonzero((got != ref).any(axis=-1))):
            row = np.sort(e_ref[b, h, i])[::-1]
            pre = np.concatenate([[0.0], np.cumsum(row)])
            k_lo, k_hi = sorted((int(got[b, h, i].sum()), int(ref[b, h, i].sum())))
            slack = 3 * E_RTOL * pre[-1]
            assert all(abs(pre[kk] - eps * pre[-1]) <= slack for kk in range(k_lo, k_hi + (k_lo == k_hi))), \
                (b, h, i, k_lo, k_hi)
            ambiguous[h, i] = True
    final = cal.finish(rho).cpu().numpy().astype(bool)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    ref_final = aggregate_masks(np.concatenate(ref_samples, axis=0), rho)
    ok = ~ambiguous
    assert np.array_equal(final[ok], ref_final[ok])
    assert ambiguous.mean() < 0.05
    density = final.mean()
    assert 0.0 < density < 1.0
