"""GPU block-mask -> CSR vs the oracle: bit-exact row_ptr, col_idx and nnz."""
import json
import os

import numpy as np
import pytest
import torch

from oracle.mask import all_mask, dense_to_csr, two_stage_mask, window_anchor_mask
from synthetic import WORKLOADS, mask_variants, static_calibrated_mask
from tests.gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _build(params, dense=None):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    nb = params.n_pad // params.block_size
    cap = lva.lva_block_mask_max_nnz(params)
    row_ptr = torch.full((params.mask_heads * nb + 1,), -5, dtype=torch.int32, device=dev)
    col_idx = torch.full((cap,), -5, dtype=torch.int32, device=dev)
    nnz = torch.zeros(1, dtype=torch.int32, device=dev)
    dm = torch.from_numpy(np.ascontiguousarray(dense, dtype=np.uint8)).to(dev) if dense is not None else None
    lva.lva_build_block_mask(params, dm, row_ptr, col_idx, nnz)
    torch.cuda.synchronize()
    rp = row_ptr.cpu().numpy()
    n = int(nnz.item())
    assert n == rp[-1]
    return rp, col_idx.cpu().numpy()[:n]


def _check(params, ref_masks, dense=None):
    rp, ci = _build(params, dense)
    rp_ref, ci_ref = dense_to_csr(ref_masks)
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(ci, ci_ref)


def test_tiny_golden():
    import block_sparse_attention_lva_b200 as lva
    g = json.load(open(os.path.join(GOLDEN, "mask_tiny.json")))
    p = lva.MaskParams(lva.LVA_MASK_WINDOW_ANCHOR, g["n_pad"], g["n_valid"], g["block_size"], 1,
                       g["unit_tokens"], g["radius"], g["num_anchors"], g["step"])
    rp, ci = _build(p)
    assert rp.tolist() == g["row_ptr"] and ci.tolist() == g["col_idx"]


def test_small_every_step():
    import block_sparse_attention_lva_b200 as lva
    w = WORKLOADS["small"]
    spec = mask_variants(w)[0]
    for s in spec["steps"]:
        p = lva.MaskParams(lva.LVA_MASK_WINDOW_ANCHOR, w.n_pad, w.n_valid, w.block_size, 1,
                           spec["unit"], spec["radius"], spec["anchors"], s)
        _check(p, window_anchor_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["radius"],
                                     spec["anchors"], s))


def test_static_and_all():
    import block_sparse_attention_lva_b200 as lva
    w = WORKLOADS["static"]
    dense = static_calibrated_mask(w)
    p = lva.MaskParams(lva.LVA_MASK_STATIC, w.n_pad, w.n_valid, w.block_size, w.H)
    _check(p, dense.astype(bool), dense)
    _check(lva.MaskParams(lva.LVA_MASK_ALL, w.n_pad, w.n_valid, w.block_size), all_mask(w.nb))


@pytest.mark.parametrize("name", ["large", "long"])
def test_sweeps(name):
    import block_sparse_attention_lva_b200 as lva
    w = WORKLOADS[name]
    for spec in mask_variants(w):
        if spec["kind"] == "window_anchor":
            p = lva.MaskParams(lva.LVA_MASK_WINDOW_ANCHOR, w.n_pad, w.n_valid, w.block_size, 1,
                               spec["unit"], spec["radius"], spec["anchors"], 0)
            ref = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["radius"],
                                     spec["anchors"], 0)
        elif spec["kind"] == "two_stage":
            p = lva.MaskParams(lva.LVA_MASK_TWO_STAGE, w.n_pad, w.n_valid, w.block_size, 1,
                               group_blocks=spec["group"])
            ref = two_stage_mask(w.nb, spec["group"])
        elif spec["kind"] == "lvsa_frames":
            from oracle.mask import lvsa_frame_mask
            p = lva.MaskParams(lva.LVA_MASK_LVSA_FRAMES, w.n_pad, w.n_valid, w.block_size, 1, spec["unit"],
                               num_anchors=spec["anchors"], step=0, budget_frames=spec["budget"])
            ref = lvsa_frame_mask(w.n_pad, w.n_valid, w.block_size, spec["unit"], spec["anchors"], 0,
                                  spec["budget"])
        else:
            p = lva.MaskParams(lva.LVA_MASK_ALL, w.n_pad, w.n_valid, w.block_size)
            ref = all_mask(w.nb)
        _check(p, ref)


def test_edge_cases():
    import block_sparse_attention_lva_b200 as lva
    rng = np.random.default_rng(9)
    # Static masks whose rows are not 16-byte multiples (byte path), with empty rows.
    for hm, nb in [(3, 37), (2, 1), (1, 600)]:
        dense = (rng.random((hm, nb, nb)) < 0.2).astype(np.uint8)
        dense[0, 0] = 0
        p = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 64, nb * 64 - 5, 64, hm)
        _check(p, dense.astype(bool), dense)
    # Static, vector path, a row entirely empty and one entirely full.
    dense = (rng.random((2, 64, 64)) < 0.5).astype(np.uint8)
    dense[1, 3] = 0
    dense[1, 4] = 1
    _check(lva.MaskParams(lva.LVA_MASK_STATIC, 64 * 128, 64 * 128, 128, 2), dense.astype(bool), dense)
    # Window masks with trailing padding-only blocks, radius 0, anchors beyond the window,
    # large step, many anchors.
    for (n_pad, n_valid, bs, U, r, G, s) in [(1024, 700, 64, 100, 0, 3, 123), (4096, 4096, 128, 128, 0, 32, 5),
                                            (8192, 5000, 128, 1560, 2, 1, 0), (640, 64, 64, 64, 1, 10, 7)]:
        p = lva.MaskParams(lva.LVA_MASK_WINDOW_ANCHOR, n_pad, n_valid, bs, 1, U, r, G, s)
        _check(p, window_anchor_mask(n_pad, n_valid, bs, U, r, G, s))
    for nb, g in [(10, 3), (7, 7), (5, 1), (9, 20)]:
        p = lva.MaskParams(lva.LVA_MASK_TWO_STAGE, nb * 128, nb * 128, 128, 1, group_blocks=g)
        _check(p, two_stage_mask(nb, g))


@pytest.mark.parametrize("n_pad,n_valid,bs,U,G,C,steps", [
    (32768, 32760, 128, 1560, 4, 8, (0, 3, 11)),       # small workload grid, 21 frames
    (126464, 126360, 128, 1560, 4, 21, (0, 5)),        # long workload grid, 81 frames, budget 21
    (256, 256, 64, 64, 1, 2, (0, 1, 2, 3)),            # tiny: one block per frame
    (6400, 6375, 128, 100, 5, 17, (0, 9)),             # frames of 100 tokens: blocks span 2-3 frames
    (4096, 4000, 128, 1000, 2, 9, (1,)),               # budget above the frame count (4 frames)
    (8192, 8192, 64, 512, 0, 5, (0,)),                 # no global frames: symmetric windows
])
def test_lvsa_frames(n_pad, n_valid, bs, U, G, C, steps):
    import block_sparse_attention_lva_b200 as lva
    from oracle.mask import lvsa_frame_mask
    for s in steps:
        p = lva.MaskParams(lva.LVA_MASK_LVSA_FRAMES, n_pad, n_valid, bs, 1, U, num_anchors=G, step=s,
                           budget_frames=C)
        _check(p, lvsa_frame_mask(n_pad, n_valid, bs, U, G, s, C))


# ---------------------------------------------------------------- packed static build (workspace)
def _build_ws(params, dense, ws_bytes=None):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    nb = params.n_pad // params.block_size
    cap = lva.lva_block_mask_max_nnz(params)
    need = lva.lva_block_mask_workspace_bytes(params)
    row_ptr = torch.full((params.mask_heads * nb + 1,), -5, dtype=torch.int32, device=dev)
    col_idx = torch.full((cap,), -5, dtype=torch.int32, device=dev)
    nnz = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.full((need if ws_bytes is None else ws_bytes,), 0xAB, dtype=torch.uint8, device=dev)
    dm = torch.from_numpy(np.ascontiguousarray(dense, dtype=np.uint8)).to(dev)
    lva.lva_build_block_mask_ws(params, dm, row_ptr, col_idx, nnz, ws)
    torch.cuda.synchronize()
    rp = row_ptr.cpu().numpy()
    n = int(nnz.item())
    assert n == rp[-1]
    return rp, col_idx.cpu().numpy()[:n]


@pytest.mark.parametrize("hm,nb,density,seed", [
    (12, 256, 0.3, 1),        # the static workload's shape: one-CTA scan
    (3, 37, 0.5, 2),          # nb not a multiple of 16: byte-wise pack
    (2, 48, 0.5, 3),          # a half-filled last word
    (20, 256, 0.2, 4),        # 5120 rows: tiled scan over several CTAs
    (5, 1000, 0.05, 5),       # 5000 rows, nb % 32 == 8
    (1, 4096, 0.3, 6),        # a 4096-block row: four 1024-column rounds per warp
])
def test_packed_static_build_matches_oracle(hm, nb, density, seed):
    import block_sparse_attention_lva_b200 as lva
    rng = np.random.default_rng(seed)
    dense = (rng.random((hm, nb, nb)) < density).astype(np.uint8) * rng.integers(1, 256, (hm, nb, nb), dtype=np.uint8)
    dense[0, 0] = 0                     # an empty row
    dense[-1, -1] = 7                   # a full row (any nonzero byte counts)
    p = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 128, nb * 128 - 5, 128, hm)
    rp, ci = _build_ws(p, dense)
    rp_ref, ci_ref = dense_to_csr(dense != 0)
    assert np.array_equal(rp, rp_ref) and np.array_equal(ci, ci_ref)


def test_packed_static_build_at_stress_scale_equals_two_read_build():
    """8 heads x 4096 x 4096 blocks (134 MB): the workspace build equals the two-read build
    bit for bit (tiled scan over 8 CTAs, 32,768 rows)."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    hm, nb = 8, 4096
    g = torch.Generator(device=dev).manual_seed(15)
    dense = (torch.rand((hm, nb, nb), generator=g, device=dev) < 0.3).to(torch.uint8)
    p = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 128, nb * 128, 128, hm)
    cap = lva.lva_block_mask_max_nnz(p)
    outs = []
    for ws in (None, torch.empty(lva.lva_block_mask_workspace_bytes(p), dtype=torch.uint8, device=dev)):
        row_ptr = torch.empty(hm * nb + 1, dtype=torch.int32, device=dev)
        col_idx = torch.empty(cap, dtype=torch.int32, device=dev)
        nnz = torch.empty(1, dtype=torch.int32, device=dev)
        if ws is None:
            lva.lva_build_block_mask(p, dense, row_ptr, col_idx, nnz)
        else:
            lva.lva_build_block_mask_ws(p, dense, row_ptr, col_idx, nnz, ws)
        torch.cuda.synchronize()
        n = int(nnz.item())
        outs.append((row_ptr.cpu(), col_idx[:n].cpu(), n))
        del col_idx
    assert outs[0][2] == outs[1][2]
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    # spot-check a few rows against the dense mask itself
    d = dense.cpu().numpy()
    rp, ci = outs[1][0].numpy(), outs[1][1].numpy()
    for r in (0, 1, 4095, 4096, 20000, hm * nb - 1):
        assert np.array_equal(ci[rp[r]:rp[r + 1]], np.nonzero(d.reshape(-1, nb)[r])[0])


def test_packed_build_argument_errors():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    nb = 64
    p = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 128, nb * 128, 128, 2)
    dense = torch.ones((2, nb, nb), dtype=torch.uint8, device=dev)
    row_ptr = torch.empty(2 * nb + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(lva.lva_block_mask_max_nnz(p), dtype=torch.int32, device=dev)
    nnz = torch.empty(1, dtype=torch.int32, device=dev)
    need = lva.lva_block_mask_workspace_bytes(p)
    with pytest.raises(lva.LvaError, match="LVA_ERR_INVALID_ARG"):
        lva.lva_build_block_mask_ws(p, dense, row_ptr, col_idx, nnz, None)
    with pytest.raises(lva.LvaError, match="LVA_ERR_CAPACITY"):
        lva.lva_build_block_mask_ws(p, dense, row_ptr, col_idx, nnz,
                                    torch.empty(need - 16, dtype=torch.uint8, device=dev))
    # parametric kinds need no workspace
    q = lva.MaskParams(lva.LVA_MASK_ALL, nb * 128, nb * 128, 128, 1)
    assert lva.lva_block_mask_workspace_bytes(q) == 0
    lva.lva_build_block_mask_ws(q, None, row_ptr, col_idx, nnz, None)
    torch.cuda.synchronize()
    assert int(nnz.item()) == nb * nb
