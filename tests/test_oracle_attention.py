"""Pins for the oracle's block-masked attention (no GPU).

Each test compares the oracle with something other than itself: a library routine
(torch's float64 scaled_dot_product_attention), the token-level brute force, a closed
form, or an invariant of softmax attention.
"""
import math

import numpy as np
import pytest
import torch

from oracle.attention import attention_blocked, attention_bruteforce
from oracle.mask import window_anchor_mask


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _inputs(B, H, n_pad, d, seed):
    return _rand((B, H, n_pad, d), seed), _rand((B, H, n_pad, d), seed + 1), _rand((B, H, n_pad, d), seed + 2)


@pytest.mark.parametrize("n_pad,n_valid,bs,hm,seed", [
    (64, 64, 16, 1, 0), (96, 83, 32, 2, 1), (128, 128, 64, 2, 2), (256, 200, 64, 1, 3),
    (512, 512, 128, 2, 4),
])
def test_blocked_equals_bruteforce(n_pad, n_valid, bs, hm, seed):
    B, H, d = 1, 2, 16
    q, k, v = _inputs(B, H, n_pad, d, seed)
    nb = n_pad // bs
    rng = np.random.default_rng(seed)
    masks = rng.random((hm, nb, nb)) < 0.4
    masks[0, 0] = False                                     # an empty row
    if nb > 2:
        masks[-1, 1] = False
        masks[-1, 1, nb - 1] = True                         # a row that may attend only padding
    scale = 1.0 / math.sqrt(d)
    o1, l1 = attention_blocked(q, k, v, masks, bs, n_valid, scale)
    o2, l2 = attention_bruteforce(q, k, v, masks, bs, n_valid, scale)
    assert np.max(np.abs(o1 - o2)) < 1e-12
    fin = np.isfinite(l2)
    assert np.array_equal(fin, np.isfinite(l1))
    assert np.max(np.abs(l1[fin] - l2[fin])) < 1e-12
    assert np.all(l1[~fin] == -np.inf) and np.all(o1[~fin] == 0.0)


@pytest.mark.parametrize("n_valid", [256, 230])
def test_all_ones_equals_library_sdpa(n_valid):
    B, H, n_pad, d, bs = 1, 3, 256, 32, 64
    q, k, v = _inputs(B, H, n_pad, d, 11)
    scale = float(np.float32(0.125))
    o, lse = attention_blocked(q, k, v, np.ones((1, 4, 4), bool), bs, n_valid, scale)
    keep = torch.arange(n_pad) < n_valid
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), attn_mask=keep[None, None, None, :].expand(B, H, n_pad, n_pad),
        scale=scale)
    assert np.max(np.abs(o - ref.numpy())) < 1e-12
    # LSE against torch.logsumexp of the scaled scores.
    s = scale * (q.double() @ k.double().transpose(-1, -2))
    s = s.masked_fill(~keep, float("-inf"))
    assert np.max(np.abs(lse - torch.logsumexp(s, dim=-1).numpy())) < 1e-12


def test_identical_keys_closed_form():
    # All keys equal k: O_r is the mean of the attended v_c, LSE_r = scale*q_r.k + ln|J|.
    B, H, n_pad, d, bs = 1, 1, 192, 8, 64
    q, _, v = _inputs(B, H, n_pad, d, 21)
    kvec = _rand((d,), 99)
    k = kvec.expand(B, H, n_pad, d).clone()
    masks = np.array([[[1, 0, 1], [0, 1, 0], [1, 1, 1]]], bool)
    n_valid = 170
    scale = 0.3
    o, lse = attention_blocked(q, k, v, masks, bs, n_valid, scale)
    qd, vd, kd = q.double().numpy(), v.double().numpy(), kvec.double().numpy()
    sc = float(np.float32(scale))
    for i in range(3):
        keys = [c for j in range(3) if masks[0, i, j] for c in range(j * bs, (j + 1) * bs) if c < n_valid]
        rows = slice(i * bs, (i + 1) * bs)
        assert np.max(np.abs(o[0, 0, rows] - vd[0, 0, keys].mean(axis=0))) < 1e-12
        exp_lse = sc * (qd[0, 0, rows] @ kd) + math.log(len(keys))
        assert np.max(np.abs(lse[0, 0, rows] - exp_lse)) < 1e-12


def test_rows_sum_to_one():
    w_pad, bs = 256, 64
    q, k, v = _inputs(1, 2, w_pad, 64, 31)
    m = window_anchor_mask(w_pad, w_pad, bs, bs, 1, 1, 0)
    _, _, probs = attention_blocked(q, k, v, m, bs, w_pad, 0.125, return_probs=True)
    for (_, _, i), (keys, p) in probs.items():
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-13
        assert np.all(p >= 0)
        assert set(keys // bs) == set(np.flatnonzero(m[i]))


def test_key_permutation_within_block_invariance():
    n_pad, bs, d = 256, 64, 16
    q, k, v = _inputs(1, 2, n_pad, d, 41)
    m = np.random.default_rng(0).random((1, 4, 4)) < 0.6
    o1, l1 = attention_blocked(q, k, v, m, bs, n_pad, 0.25)
    perm = torch.arange(n_pad)
    g = torch.Generator().manual_seed(7)
    for j in range(4):
        perm[j * bs:(j + 1) * bs] = j * bs + torch.randperm(bs, generator=g)
    o2, l2 = attention_blocked(q, k[:, :, perm], v[:, :, perm], m, bs, n_pad, 0.25)
    fin = np.isfinite(l1)
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l1[fin] - l2[fin])) < 1e-12


def test_key_offset_shifts_lse_only():
    n_pad, bs, d = 128, 32, 16
    q, k, v = _inputs(1, 1, n_pad, d, 51)
    m = np.random.default_rng(1).random((1, 4, 4)) < 0.7
    np.fill_diagonal(m[0], True)
    c = torch.full((d,), 0.5, dtype=torch.float64)
    scale = 0.25
    o1, l1 = attention_blocked(q, k, v, m, bs, n_pad, scale)
    o2, l2 = attention_blocked(q.double(), k.double() + c, v.double(), m, bs, n_pad, scale)
    shift = scale * (q.double().numpy()[0, 0] @ c.numpy())
    assert np.max(np.abs(o1 - o2)) < 1e-12
    assert np.max(np.abs(l2[0, 0] - l1[0, 0] - shift)) < 1e-12


def test_single_active_key():
    # Only the last block is active and it holds one real token: O_r = v_c, LSE_r = s_c.
    n_pad, bs, d = 128, 64, 8
    n_valid = 65
    q, k, v = _inputs(1, 1, n_pad, d, 61)
    m = np.array([[[0, 1], [0, 1]]], bool)
    scale = 0.5
    o, lse = attention_blocked(q, k, v, m, bs, n_valid, scale)
    qd, kd, vd = (t.double().numpy()[0, 0] for t in (q, k, v))
    assert np.max(np.abs(o[0, 0] - vd[64])) < 1e-15
    assert np.max(np.abs(lse[0, 0] - scale * (qd @ kd[64]))) < 1e-12


def test_hand_worked_two_keys():
    # q = (1, 0); keys (1, 0), (0, 1); scale 1: scores (1, 0).
    q = torch.tensor([[[[1.0, 0.0]]]])
    k = torch.tensor([[[[1.0, 0.0], [0.0, 1.0]]]])
    v = torch.tensor([[[[2.0, -1.0], [0.0, 4.0]]]])
    q = torch.cat([q, torch.zeros(1, 1, 1, 2)], dim=2)      # second query row (zeros)
    o, lse = attention_blocked(q, k, v, np.ones((1, 1, 1), bool), 2, 2, 1.0)
    e = math.e
    assert np.allclose(o[0, 0, 0], [(2 * e + 0) / (e + 1), (-e + 4) / (e + 1)], atol=1e-15)
    assert abs(lse[0, 0, 0] - math.log(e + 1)) < 1e-15
    assert np.allclose(o[0, 0, 1], [1.0, 1.5], atol=1e-15) and abs(lse[0, 0, 1] - math.log(2)) < 1e-15


def test_padded_keys_never_matter():
    # Changing K/V rows beyond n_valid leaves every output unchanged.
    n_pad, bs, d, n_valid = 192, 64, 16, 150
    q, k, v = _inputs(1, 2, n_pad, d, 71)
    m = np.ones((1, 3, 3), bool)
    o1, l1 = attention_blocked(q, k, v, m, bs, n_valid, 0.25)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, n_valid:] = 30.0
    v2[:, :, n_valid:] = -7.0
    o2, l2 = attention_blocked(q, k2, v2, m, bs, n_valid, 0.25)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_broadcast_identity_map_is_plain_attention():
    from oracle.attention import attention_with_broadcast
    n_pad, bs, d = 256, 64, 16
    q, k, v = _inputs(1, 2, n_pad, d, 81)
    m = np.random.default_rng(2).random((2, 4, 4)) < 0.6
    ident = np.tile(np.arange(4, dtype=np.int32), (2, 1))
    o1, l1 = attention_with_broadcast(q, k, v, m, bs, n_pad, 0.25, ident)
    o2, l2 = attention_blocked(q, k, v, m, bs, n_pad, 0.25)
    assert np.array_equal(np.nan_to_num(o1), np.nan_to_num(o2)) and np.array_equal(l1, l2)


def test_broadcast_is_exact_when_rows_truly_repeat():
    # CalibAtt: replicating anchor rows is exact when the repeated rows really repeat.  Give
    # block 3 the queries and the key list of block 1: its output must equal the full result.
    from oracle.attention import attention_with_broadcast
    n_pad, bs, d = 256, 64, 16
    q, k, v = _inputs(1, 1, n_pad, d, 91)
    q[:, :, 3 * bs:4 * bs] = q[:, :, 1 * bs:2 * bs]
    m = np.random.default_rng(3).random((1, 4, 4)) < 0.7
    m[0, 1, 1] = True
    m[0, 3] = m[0, 1]
    src = np.array([[0, 1, 2, 1]], dtype=np.int32)
    o1, l1 = attention_with_broadcast(q, k, v, m, bs, n_pad, 0.25, src)
    o2, l2 = attention_blocked(q, k, v, m, bs, n_pad, 0.25)
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l1 - l2)) < 1e-12


def test_broadcast_source_must_be_an_anchor():
    from oracle.attention import attention_with_broadcast
    q, k, v = _inputs(1, 1, 192, 8, 5)
    with pytest.raises(AssertionError):
        attention_with_broadcast(q, k, v, np.ones((1, 3, 3), bool), 64, 192, 0.3, np.array([[1, 2, 2]]))


# ---------------------------------------------------------------- SQuad two-stage operator
def _sdpa64(q, k, v, scale, mask=None):
    return torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                            attn_mask=mask, scale=scale).numpy()


def test_squad_one_window_is_dense_attention():
    # w = n: one window, and every global group is a single token (attends itself).
    from oracle.attention import squad_two_pass
    q, k, v = _inputs(1, 2, 64, 16, 101)
    o, _ = squad_two_pass(q, k, v, 64, 0.25)
    assert np.max(np.abs(o - _sdpa64(q, k, v, 0.25))) < 1e-12


def test_squad_unit_windows_is_dense_attention():
    # w = 1: the local pass returns V, the global pass is dense attention over all tokens.
    from oracle.attention import squad_two_pass
    q, k, v = _inputs(1, 2, 48, 8, 103)
    o, o_local = squad_two_pass(q, k, v, 1, 0.3)
    assert np.max(np.abs(o_local - v.double().numpy())) < 1e-15
    assert np.max(np.abs(o - _sdpa64(q, k, v, float(np.float32(0.3))))) < 1e-12


def test_squad_matches_explicit_masked_matrices():
    # Twin: the two passes as dense masked attention (library SDPA with boolean masks).
    from oracle.attention import squad_two_pass
    n, w = 96, 8
    q, k, v = _inputs(1, 1, n, 16, 107)
    idx = torch.arange(n)
    local = (idx[:, None] // w) == (idx[None, :] // w)
    glob = (idx[:, None] % w) == (idx[None, :] % w)
    o_l = _sdpa64(q, k, v, 0.25, local)
    o_ref = _sdpa64(q, k, torch.from_numpy(o_l), 0.25, glob)
    o, o_local = squad_two_pass(q, k, v, w, 0.25)
    assert np.max(np.abs(o_local - o_l)) < 1e-12 and np.max(np.abs(o - o_ref)) < 1e-12


def test_squad_full_receptive_field():
    # Composition recovers a full receptive field: every output depends on every value row.
    from oracle.attention import squad_two_pass
    n, w = 36, 6
    q, k, v = _inputs(1, 1, n, 8, 109)
    base, _ = squad_two_pass(q, k, v, w, 0.5)
    for c in (0, 17, 35):
        v2 = v.double().clone()
        v2[0, 0, c] += 1.0
        o2, _ = squad_two_pass(q, k, v2, w, 0.5)
        assert np.all(np.abs(o2 - base).max(axis=-1) > 0)
