"""GPU block-sparse attention vs the FP64 oracle.

* Multi-tile shapes with ragged tails, empty rows, random pad contents, both head dims and
  both block sizes: every output element compared.
* The five workloads at full size through the whole layer path (reorder, CSR, attention,
  inverse reorder): every element of O and LSE for the small workload (step 0) and the
  static 30 % masks; sampled query blocks for every other mask, every row checked for
  NaN / -inf.
"""
import math

import numpy as np
import pytest
import torch

from oracle.attention import attention_blocked
from oracle.mask import all_mask, dense_to_csr, lvsa_frame_mask, two_stage_mask, window_anchor_mask
from oracle.reorder import reorder_forward, reorder_inverse, tile_permutation
from synthetic import WORKLOADS, make_qkv, mask_variants, static_calibrated_mask
from tests.gpu_helpers import check_o_lse, require_gpu

pytestmark = pytest.mark.gpu


def _rand_bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _attn_gpu(q, k, v, masks, bs, n_valid, scale):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    B, H, n_pad, d = q.shape
    rp, ci = dense_to_csr(masks)
    row_ptr = torch.from_numpy(rp).to(dev)
    col_idx = torch.from_numpy(ci if ci.size else np.zeros(1, np.int32)).to(dev)
    o = torch.full((B, H, n_pad, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, n_pad), float("nan"), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_attn(q.to(dev), k.to(dev), v.to(dev), o, lse, n_valid, bs, row_ptr,
                              col_idx[:max(ci.size, 0)] if ci.size else col_idx[:0], masks.shape[0], scale)
    torch.cuda.synchronize()
    status, detail = lva.lva_device_error()
    assert status == 0, (status, detail)
    return o, lse


@pytest.mark.parametrize("B,H,n_pad,n_valid,d,bs,hm,density,seed", [
    (1, 2, 1280, 1200, 128, 128, 2, 0.4, 0),
    (2, 3, 640, 640, 128, 128, 1, 0.6, 1),
    (1, 2, 1024, 1000, 64, 128, 2, 0.5, 2),
    (1, 2, 768, 700, 128, 64, 2, 0.3, 3),
    (1, 1, 512, 512, 64, 64, 1, 1.0, 4),
    (1, 2, 4096, 4096, 128, 128, 2, 1.0, 5),
    (1, 1, 384, 1, 128, 128, 1, 1.0, 6),
    (1, 2, 256, 0, 128, 128, 1, 1.0, 7),     # every key is padding: all rows empty
])
def test_against_oracle_full(B, H, n_pad, n_valid, d, bs, hm, density, seed):
    q = _rand_bf16((B, H, n_pad, d), seed)
    k = _rand_bf16((B, H, n_pad, d), seed + 100)
    v = _rand_bf16((B, H, n_pad, d), seed + 200)
    k[:, :, n_valid:] = 40.0                 # padded keys must never be attended
    nb = n_pad // bs
    rng = np.random.default_rng(seed)
    masks = rng.random((hm, nb, nb)) < density
    if density < 1.0:
        masks[0, 0] = False                  # empty row -> O = 0, LSE = -inf
        masks[-1, nb - 1] = True             # a full row
    scale = 1.0 / math.sqrt(d)
    o, lse = _attn_gpu(q, k, v, masks, bs, n_valid, scale)
    o_ref, lse_ref = attention_blocked(q, k, v, masks, bs, n_valid, scale)
    check_o_lse(o, lse, o_ref, lse_ref, f"shape {(B, H, n_pad, d, bs)}")



@pytest.mark.parametrize("d,bs", [(128, 128), (64, 64)])
def test_o_at_16_but_not_32_byte_alignment(d, bs):
    """O rows are written with 32-byte stores when O starts on a 32-byte boundary and with
    16-byte stores otherwise (16 bytes is the API's alignment rule): an O buffer that starts
    16 bytes past a 32-byte boundary gets the same values, bit for bit."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    B, H, n_pad, n_valid = 1, 2, 4 * bs, 4 * bs - 3
    q, k, v = (_rand_bf16((B, H, n_pad, d), 900 + t).to(dev) for t in range(3))
    nb = n_pad // bs
    masks = np.random.default_rng(9).random((1, nb, nb)) < 0.6
    masks[0, :, 0] = True
    rp, ci = dense_to_csr(masks)
    row_ptr, col_idx = torch.from_numpy(rp).to(dev), torch.from_numpy(ci).to(dev)
    scale = 1.0 / math.sqrt(d)
    outs = []
    for shift in (0, 8):                       # elements: 0 or 16 bytes past the allocation
        buf = torch.full((B * H * n_pad * d + 16,), float("nan"), dtype=torch.bfloat16, device=dev)
        o = buf[shift:shift + B * H * n_pad * d].view(B, H, n_pad, d)
        assert (o.data_ptr() % 32 == 0) == (shift == 0)
        lse = torch.empty((B, H, n_pad), dtype=torch.float32, device=dev)
        lva.lva_block_sparse_attn(q, k, v, o, lse, n_valid, bs, row_ptr, col_idx, 1, scale)
        torch.cuda.synchronize()
        assert lva.lva_device_error() == (0, 0)
        outs.append((o.clone(), lse.clone()))
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1], outs[1][1])

@pytest.mark.parametrize("d,bs", [(128, 128), (64, 64)])
def test_all_rows_empty(d, bs):
    """An empty CSR (no entries at all): every row gives O = 0 and LSE = -inf."""
    B, H, n_pad = 2, 3, 1024
    q, k, v = (_rand_bf16((B, H, n_pad, d), 70 + t) for t in range(3))
    masks = np.zeros((H, n_pad // bs, n_pad // bs), dtype=bool)
    o, lse = _attn_gpu(q, k, v, masks, bs, n_pad - 5, 1.0 / math.sqrt(d))
    assert torch.count_nonzero(o.float().cpu()).item() == 0
    assert bool(torch.all(lse.cpu() == float("-inf")))


def test_many_items_mixed_rows():
    # 2 x 8 heads x 32 query blocks = 512 work items (more than one wave of CTAs), per-head
    # masks with empty rows, single-block rows and full rows interleaved.
    B, H, n_pad, d, bs = 2, 8, 4096, 128, 128
    n_valid = 4000
    q = _rand_bf16((B, H, n_pad, d), 71)
    k = _rand_bf16((B, H, n_pad, d), 72)
    v = _rand_bf16((B, H, n_pad, d), 73)
    nb = n_pad // bs
    rng = np.random.default_rng(7)
    masks = rng.random((H, nb, nb)) < rng.random((H, nb, 1))        # row densities 0..1
    masks[:, ::7] = False                                            # empty rows
    masks[:, 3::11] = False
    masks[:, 3::11, 5] = True                                        # one block only
    masks[:, 1::13] = True                                           # full rows
    o, lse = _attn_gpu(q, k, v, masks, bs, n_valid, 1.0 / math.sqrt(d))
    o_ref, lse_ref = attention_blocked(q, k, v, masks, bs, n_valid, 1.0 / math.sqrt(d))
    check_o_lse(o, lse, o_ref, lse_ref, "many items")


def test_tiny_workload():
    w = WORKLOADS["tiny"]
    spec = mask_variants(w)[0]
    q, k, v = make_qkv(w)
    pad = w.n_pad - w.n_valid
    assert pad == 0
    m = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["radius"], spec["anchors"], 0)
    o, lse = _attn_gpu(q, k, v, m[None], w.block_size, w.n_valid, w.scale)
    o_ref, lse_ref = attention_blocked(q, k, v, m, w.block_size, w.n_valid, w.scale)
    check_o_lse(o, lse, o_ref, lse_ref, "tiny")


def test_corrupt_csr_is_reported_not_faulted():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    B, H, n_pad, d, bs = 1, 1, 512, 128, 128
    q, k, v = (_rand_bf16((B, H, n_pad, d), s) for s in (1, 2, 3))
    row_ptr = torch.tensor([0, 2, 3, 3, 5], dtype=torch.int32, device=dev)
    col_idx = torch.tensor([0, 1, 9, 2, 3], dtype=torch.int32, device=dev)   # 9 >= nb in row 1
    o = torch.empty((B, H, n_pad, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, n_pad), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_attn(q.to(dev), k.to(dev), v.to(dev), o, lse, n_pad, bs, row_ptr, col_idx, 1, 0.1)
    status, detail = lva.lva_device_error()
    assert status == 1 and detail == 1
    assert torch.all(o[0, 0, 128:256] == 0) and torch.all(torch.isneginf(lse[0, 0, 128:256]))
    m = np.zeros((1, 4, 4), bool)
    m[0, 0, [0, 1]] = True
    m[0, 3, [2, 3]] = True
    o_ref, lse_ref = attention_blocked(q, k, v, m, bs, n_pad, 0.1)
    keep = np.r_[0:128, 256:512]
    check_o_lse(o[:, :, keep], lse[:, :, keep], o_ref[:, :, keep], lse_ref[:, :, keep], "corrupt csr")
    # row_ptr pointing past col_len is rejected the same way (the only fault of this call:
    # the first fault recorded wins, so no other row may be corrupt)
    row_ptr2 = torch.tensor([0, 2, 3, 3, 50], dtype=torch.int32, device=dev)
    col_idx2 = torch.tensor([0, 1, 1, 2, 3], dtype=torch.int32, device=dev)
    lva.lva_block_sparse_attn(q.to(dev), k.to(dev), v.to(dev), o, lse, n_pad, bs, row_ptr2, col_idx2, 1, 0.1)
    status, detail = lva.lva_device_error()
    assert status == 1 and detail == 3


def test_repeated_column_is_reported_not_counted_twice():
    """A CSR row that lists a key block twice (not strictly ascending) is skipped and
    reported, never attended twice."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    B, H, n_pad, d, bs = 1, 1, 512, 128, 128
    q, k, v = (_rand_bf16((B, H, n_pad, d), s) for s in (11, 12, 13))
    row_ptr = torch.tensor([0, 2, 4, 6, 8], dtype=torch.int32, device=dev)
    col_idx = torch.tensor([0, 1, 2, 2, 1, 3, 0, 3], dtype=torch.int32, device=dev)   # row 1 repeats 2
    o = torch.empty((B, H, n_pad, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, n_pad), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_attn(q.to(dev), k.to(dev), v.to(dev), o, lse, n_pad, bs, row_ptr, col_idx, 1, 0.1)
    status, detail = lva.lva_device_error()
    assert status == 1 and detail == 1
    assert torch.all(o[0, 0, 128:256] == 0) and torch.all(torch.isneginf(lse[0, 0, 128:256]))
    m = np.zeros((1, 4, 4), bool)
    m[0, 0, [0, 1]] = True
    m[0, 2, [1, 3]] = True
    m[0, 3, [0, 3]] = True
    o_ref, lse_ref = attention_blocked(q, k, v, m, bs, n_pad, 0.1)
    keep = np.r_[0:128, 256:512]
    check_o_lse(o[:, :, keep], lse[:, :, keep], o_ref[:, :, keep], lse_ref[:, :, keep], "repeated column")


@pytest.mark.parametrize("B,H,n_pad,n_valid,d,bs,hm,density,seed", [
    (1, 3, 2048, 2000, 128, 128, 3, 0.5, 21),
    (2, 2, 1024, 1024, 64, 128, 1, 1.0, 22),
    (1, 2, 768, 700, 128, 64, 2, 0.4, 23),
])
def test_lse_only_matches_attention_lse(B, H, n_pad, n_valid, d, bs, hm, density, seed):
    """lva_block_sparse_lse gives the LSE of lva_block_sparse_attn (same scores and maxima;
    sums within the exponential split's error) and matches the oracle; empty rows give -inf."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    q, k, v = (_rand_bf16((B, H, n_pad, d), seed + 100 * t) for t in range(3))
    nb = n_pad // bs
    masks = np.random.default_rng(seed).random((hm, nb, nb)) < density
    masks[0, 1] = False                                      # an empty row
    scale = 1.0 / math.sqrt(d)
    _, lse_full = _attn_gpu(q, k, v, masks, bs, n_valid, scale)
    rp, ci = dense_to_csr(masks)
    lse = torch.full((B, H, n_pad), float("nan"), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_lse(q.to(dev), k.to(dev), lse, n_valid, bs, torch.from_numpy(rp).to(dev),
                             torch.from_numpy(ci).to(dev), hm, scale)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    a, b = lse.cpu().numpy(), lse_full.cpu().numpy()
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    fin = np.isfinite(b)
    # The two forms send different exponential pairs to the FMA-pipe polynomial (relative
    # error <= 7.5e-5, tests/test_exp2_poly.py) and the rest to ex2.approx, so their row sums
    # differ by at most that relative error and their LSEs by at most ~7.5e-5.
    assert np.abs(a[fin] - b[fin]).max() <= 1e-4
    _, lse_ref = attention_blocked(q, k, v, masks, bs, n_valid, scale)
    assert np.array_equal(np.isneginf(a), np.isneginf(lse_ref))
    assert np.abs(a[fin] - lse_ref[fin]).max() <= 1e-3



@pytest.mark.parametrize("d,bs,n_pad,n_valid,seed", [(128, 128, 1280, 1200, 31), (64, 64, 768, 700, 32)])
def test_negative_scale(d, bs, n_pad, n_valid, seed):
    """A negative softmax scale (the row max of scale * s is scale * min s) runs its own
    kernel instantiation: every element of O and LSE, and the LSE-only form, match the
    oracle; padded keys (scores that would dominate if attended) stay excluded."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    q, k, v = (_rand_bf16((1, 2, n_pad, d), seed + 100 * t) for t in range(3))
    k[:, :, n_valid:] = -40.0
    nb = n_pad // bs
    masks = np.random.default_rng(seed).random((2, nb, nb)) < 0.5
    masks[0, 0] = False
    masks[-1, nb - 1] = True
    scale = -1.0 / math.sqrt(d)
    o, lse = _attn_gpu(q, k, v, masks, bs, n_valid, scale)
    o_ref, lse_ref = attention_blocked(q, k, v, masks, bs, n_valid, scale)
    check_o_lse(o, lse, o_ref, lse_ref, f"negative scale {(n_pad, d, bs)}")
    rp, ci = dense_to_csr(masks)
    lse_only = torch.full((1, 2, n_pad), float("nan"), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_lse(q.to(dev), k.to(dev), lse_only, n_valid, bs, torch.from_numpy(rp).to(dev),
                             torch.from_numpy(ci).to(dev), 2, scale)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    a = lse_only.cpu().numpy()
    assert np.array_equal(np.isneginf(a), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    assert np.abs(a[fin] - lse_ref[fin]).max() <= 1e-3


@pytest.mark.parametrize("d,bs,grow_rows", [(128, 128, "all"), (128, 128, "some"), (64, 64, "some")])
def test_running_max_jumps_take_the_redo_path(d, bs, grow_rows):
    """Key blocks after a row's first whose scores exceed the running reference by far more
    than the lazy-rescale threshold: the speculative step must give the block up and the
    max-first step redo it (with the O rescale).  Every element of O and LSE, and the
    LSE-only form, match the oracle -- for jumps in every row, and in some rows only (so
    that some warps redo a block and others commit it)."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    B, H, n_pad, n_valid = 1, 2, 8 * bs, 8 * bs - 9
    q, k, v = (_rand_bf16((B, H, n_pad, d), 700 + t) for t in range(3))
    nb = n_pad // bs
    # Queries share a component along a unit vector u, and the keys of blocks 3 and 6 carry a
    # large multiple of u: in (nearly) every row the block max of scale * s grows by more
    # than 8 in log2 units at block 3 and again at block 6.  With "some", only the queries of
    # even 16-row groups carry the component.
    u = torch.randn(d, generator=torch.Generator().manual_seed(77))
    u = u / u.norm()
    cq = torch.full((n_pad,), 4.0)
    if grow_rows == "some":
        cq[(torch.arange(n_pad) // 16) % 2 == 1] = 0.0
    q = (q.float() + cq[None, None, :, None] * u).to(torch.bfloat16)
    for jb, amp in ((3, 3.0), (6, 6.0)):
        k[:, :, jb * bs:(jb + 1) * bs] = (k[:, :, jb * bs:(jb + 1) * bs].float() + amp * math.sqrt(d) * u).to(torch.bfloat16)
    masks = np.ones((1, nb, nb), dtype=bool)
    scale = 1.0 / math.sqrt(d)
    o, lse = _attn_gpu(q, k, v, masks, bs, n_valid, scale)
    o_ref, lse_ref = attention_blocked(q, k, v, masks, bs, n_valid, scale)
    check_o_lse(o, lse, o_ref, lse_ref, f"max jumps {(d, bs, grow_rows)}")
    rp, ci = dense_to_csr(masks)
    lse_only = torch.full((B, H, n_pad), float("nan"), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_lse(q.to(dev), k.to(dev), lse_only, n_valid, bs, torch.from_numpy(rp).to(dev),
                             torch.from_numpy(ci).to(dev), 1, scale)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    a = lse_only.cpu().numpy()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(a), fin)
    assert np.abs(a[fin] - lse_ref[fin]).max() <= 1e-3

# ---------------------------------------------------------------- full workloads
def _oracle_mask(w, spec, step):
    if spec["kind"] == "window_anchor":
        return window_anchor_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["radius"],
                                  spec["anchors"], step)[None]
    if spec["kind"] == "two_stage":
        return two_stage_mask(w.nb, spec["group"])[None]
    if spec["kind"] == "all":
        return all_mask(w.nb)[None]
    if spec["kind"] == "lvsa_frames":
        return lvsa_frame_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["anchors"], step,
                               spec["budget"])[None]
    return static_calibrated_mask(w).astype(bool)


def _sample_blocks(w, masks, seed, per_head=2):
    rng = np.random.default_rng(seed)
    out = []
    for h in range(w.H):
        picks = {0, w.nb - 1} if h % 3 == 0 else set()
        picks |= set(rng.integers(0, w.nb, size=per_head).tolist())
        out += [(h, i) for i in sorted(picks)]
    return out


def _run_workload(name, labels, steps=(0,), per_head=2, whole=False):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    P = w.B * w.H
    # tile-order inputs for the oracle, by the oracle's own reorder (bit copies)
    tile = [torch.from_numpy(reorder_forward(x.view(torch.int16).reshape(P, w.n_valid, w.d).numpy(), perm,
                                             w.n_pad)).view(torch.bfloat16).reshape(w.B, w.H, w.n_pad, w.d)
            for x in (q, k, v)]
    for spec in mask_variants(w):
        if spec["label"] not in labels:
            continue
        static = static_calibrated_mask(w) if spec["kind"] == "static" else None
        layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                              static_mask=static, scale=w.scale, device=dev)
        for s in steps:
            o, lse = layer(qd, kd, vd, step=s)
            torch.cuda.synchronize()
            status, detail = lva.lva_device_error()
            assert status == 0, (status, detail)
            masks = _oracle_mask(w, spec, s)
            rp, ci = dense_to_csr(masks)
            assert np.array_equal(layer.row_ptr.cpu().numpy(), rp)
            assert np.array_equal(layer.col_idx[:ci.size].cpu().numpy(), ci)
            # every row: no NaN, LSE finite (every row of these masks is non-empty)
            assert not torch.isnan(o).any()
            assert torch.isfinite(layer.lse).all()
            lse_t = layer.lse.cpu().numpy()
            o_r = o.float().cpu().numpy()
            if whole:
                # every element of O (raster order) and LSE (tile order), all heads and rows
                ro, rl = attention_blocked(tile[0], tile[1], tile[2], masks, w.block_size, w.n_valid, w.scale)
                ro_raster = reorder_inverse(ro.reshape(P, w.n_pad, w.d), perm).reshape(o_r.shape)
                check_o_lse(o_r, lse_t, ro_raster, rl, f"{name}/{spec['label']}/s{s} (every element)")
                continue
            got_o, got_l, ref_o, ref_l = [], [], [], []
            for h, i in _sample_blocks(w, masks, seed=w.seed * 100 + s, per_head=per_head):
                hm = h if masks.shape[0] > 1 else 0
                ro, rl = attention_blocked(tile[0][:, h:h + 1], tile[1][:, h:h + 1], tile[2][:, h:h + 1],
                                           masks[hm:hm + 1], w.block_size, w.n_valid, w.scale,
                                           query_blocks=[(0, 0, i)])
                rows = np.arange(i * w.block_size, (i + 1) * w.block_size)
                real = rows[rows < w.n_valid]
                # O comes back in raster order: tile-order row r sits at raster position perm[r]
                ref_o.append(ro[0, 0, real]); got_o.append(o_r[0, h, perm[real]])
                ref_l.append(rl[0, 0, rows]); got_l.append(lse_t[0, h, rows])
            check_o_lse(np.concatenate(got_o), np.concatenate(got_l), np.concatenate(ref_o),
                        np.concatenate(ref_l), f"{name}/{spec['label']}/s{s}")



def test_workload_small():
    _run_workload("small", {"frame1_anchor4"}, steps=(1, 37, 49))


def test_workload_small_every_element():
    """The small workload at step 0: every element of O and LSE against the oracle."""
    _run_workload("small", {"frame1_anchor4"}, steps=(0,), whole=True)


def test_workload_static():
    _run_workload("static", {"all"})


def test_workload_static30_every_element():
    """Per-head static 30 % masks: every element of O and LSE against the oracle."""
    _run_workload("static", {"static30"}, whole=True)


def test_workload_large():
    _run_workload("large", {"band28_anchor4", "band60_anchor4", "band171_anchor4"}, per_head=1)


def test_workload_long():
    _run_workload("long", {"two_stage", "band23_anchor4", "band48_anchor4", "band130_anchor4",
                           "band287_anchor4", "all", "lvsa_c21_g4"}, per_head=1)


@pytest.mark.parametrize("name,grid,tile,d,bs", [
    ("small", None, None, None, None),                       # 8 padded rows, partial edge tiles
    ("ragged", (3, 10, 21), (1, 4, 8), 128, 128),           # 630 tokens: partial tiles everywhere
    ("d64bs64", (2, 9, 13), (2, 3, 5), 64, 64),             # depth-2 tiles, last slab partial
])
def test_fused_raster_output_matches_separate_reorder(name, grid, tile, d, bs):
    """lva_block_sparse_attn_raster == lva_block_sparse_attn followed by the inverse reorder,
    bit for bit (the same kernel rows, only the store address differs)."""
    import block_sparse_attention_lva_b200 as lva
    from synthetic import Workload
    dev = require_gpu()
    if grid is None:
        w = WORKLOADS[name]
    else:
        w = Workload(name, B=1, H=3, d=d, T=grid[0], Hg=grid[1], Wg=grid[2], tile=tile, block_size=bs, seed=41)
    q, k, v = make_qkv(w)
    spec = dict(kind="window_anchor", unit=w.Hg * w.Wg, radius=1, anchors=2)
    layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                          scale=w.scale, device=dev)
    layer.reorder_in(q.to(dev), k.to(dev), v.to(dev))
    layer.build_mask(1)
    layer.attend()
    layer.reorder_out()
    o_sep, lse_sep = layer.o.clone(), layer.lse.clone()
    layer.o.fill_(float("nan"))
    layer.lse.fill_(float("nan"))
    layer.attend_to_raster()
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    from tests.gpu_helpers import bits
    assert np.array_equal(bits(layer.o), bits(o_sep))
    assert np.array_equal(bits(layer.lse), bits(lse_sep))


@pytest.mark.parametrize("d,bs,hm,with_src", [(128, 128, 1, False), (128, 128, 3, True), (64, 64, 3, False)])
def test_multi_block_ctas_match_single_block_ctas(d, bs, hm, with_src):
    """Short rows passed with their exact entry count run CTAs that walk 4 query blocks each;
    the same CSR passed with a larger capacity runs one query block per CTA.  Same rows, same
    arithmetic: the outputs must agree bit for bit (including empty rows and skipped blocks)."""
    import block_sparse_attention_lva_b200 as lva
    from tests.gpu_helpers import bits
    dev = require_gpu()
    B, H = 1, 3
    n_pad = 64 * bs
    n_valid = n_pad - 37                                     # a ragged tail
    nb = n_pad // bs
    q, k, v = (_rand_bf16((B, H, n_pad, d), s) for s in (11, 12, 13))
    rng = np.random.default_rng(d + bs + hm)
    masks = rng.random((hm, nb, nb)) < 0.04                  # ~2.6 key blocks per row
    masks[0, 5] = False                                      # an empty row
    rp, ci = dense_to_csr(masks)
    row_ptr = torch.from_numpy(rp).to(dev)
    exact = torch.from_numpy(ci).to(dev)
    padded = torch.zeros(hm * nb * nb, dtype=torch.int32, device=dev)
    padded[:ci.size] = exact
    src = None
    if with_src:
        s_ = np.tile(np.arange(nb, dtype=np.int32), (H, 1))
        s_[1, 1::2] = np.arange(0, nb, 2, dtype=np.int32)   # head 1: odd blocks copy the even one before
        src = torch.from_numpy(s_).to(dev)
    outs = []
    for col in (exact, padded):
        o = torch.full((B, H, n_pad, d), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full((B, H, n_pad), float("nan"), dtype=torch.float32, device=dev)
        lva.lva_block_sparse_attn(q.to(dev), k.to(dev), v.to(dev), o, lse, n_valid, bs, row_ptr, col, hm,
                                  d ** -0.5, src)
        torch.cuda.synchronize()
        assert lva.lva_device_error() == (0, 0)
        outs.append((o, lse))
    assert np.array_equal(bits(outs[0][0]), bits(outs[1][0]))
    assert np.array_equal(bits(outs[0][1]), bits(outs[1][1]))
    # and against the oracle for the computed blocks
    o_ref, lse_ref = attention_blocked(q, k, v, masks, bs, n_valid, d ** -0.5)
    computed = np.ones((H, nb), bool) if src is None else (src.cpu().numpy() == np.arange(nb))
    for h in range(H):
        rows = np.concatenate([np.arange(i * bs, (i + 1) * bs) for i in range(nb) if computed[h, i]])
        check_o_lse(outs[0][0][:, h:h + 1, rows], outs[0][1][:, h:h + 1, rows], o_ref[:, h:h + 1, rows],
                    lse_ref[:, h:h + 1, rows], f"head {h}")
