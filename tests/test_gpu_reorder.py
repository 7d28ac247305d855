"""GPU reorder vs the oracle's tile permutation: bit-exact."""
import numpy as np
import pytest
import torch

from oracle.reorder import reorder_forward, reorder_inverse, tile_permutation
from synthetic import WORKLOADS
from tests.gpu_helpers import bits, require_gpu

pytestmark = pytest.mark.gpu


def _run(grid, tile, planes, row, n_pad, dtype=torch.bfloat16, seed=0):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    T, H, W = grid
    n = T * H * W
    g = torch.Generator().manual_seed(seed)
    if dtype == torch.bfloat16:
        src = torch.randint(-2**15, 2**15, (planes, n, row), generator=g, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    else:
        src = torch.randint(-2**31, 2**31 - 1, (planes, n, row), generator=g, dtype=torch.int64).to(torch.int32).view(dtype)
    src_d = src.to(dev)
    fwd = torch.full((planes, n_pad, row), 7, dtype=dtype, device=dev)   # pad rows must be zeroed
    lva.lva_reorder_tokens(src_d, fwd, grid, tile, n_pad, inverse=False)
    back = torch.empty((planes, n, row), dtype=dtype, device=dev)
    lva.lva_reorder_tokens(fwd, back, grid, tile, n_pad, inverse=True)
    torch.cuda.synchronize()
    perm = tile_permutation(T, H, W, *tile)
    ref = reorder_forward(bits(src), perm, n_pad)
    assert np.array_equal(bits(fwd), ref)
    assert np.array_equal(bits(back), bits(src))
    assert np.array_equal(reorder_inverse(ref, perm), bits(src))


@pytest.mark.parametrize("name", ["tiny", "small", "large", "long"])
def test_workload_shapes(name):
    w = WORKLOADS[name]
    planes = min(w.B * w.H, 4)
    _run((w.T, w.Hg, w.Wg), w.tile, planes, w.d, w.n_pad, seed=w.seed)


@pytest.mark.parametrize("grid,tile,planes,row,n_pad,dtype", [
    ((3, 5, 7), (2, 2, 4), 3, 64, 128, torch.bfloat16),     # partial tiles in t, h and w
    ((5, 9, 11), (2, 4, 4), 5, 3, 512, torch.bfloat16),     # 6-byte rows (2-byte accesses)
    ((2, 6, 10), (1, 4, 8), 7, 4, 128, torch.bfloat16),     # 8-byte rows
    ((4, 8, 8), (1, 8, 16), 2, 1, 256, torch.float32),      # tile wider than the grid; 4-byte rows (LSE-like)
    ((1, 1, 1), (1, 1, 1), 1, 8, 64, torch.bfloat16),       # one token
])
def test_odd_shapes(grid, tile, planes, row, n_pad, dtype):
    _run(grid, tile, planes, row, n_pad, dtype)


def test_iota_returns_permutation():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    w = WORKLOADS["small"]
    n = w.n_valid
    iota = torch.arange(n, dtype=torch.int32, device=dev).view(1, n, 1).view(torch.float32)
    out = torch.empty((1, w.n_pad, 1), dtype=torch.float32, device=dev)
    lva.lva_reorder_tokens(iota, out, (w.T, w.Hg, w.Wg), w.tile, w.n_pad)
    got = out.view(torch.int32).cpu().numpy()[0, :, 0]
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    assert np.array_equal(got[:n], perm) and np.all(got[n:] == 0)


def test_stacked_qkv_single_launch_matches_separate():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    w = WORKLOADS["small"]
    g = torch.Generator().manual_seed(3)
    qkv = torch.randint(-2**15, 2**15, (3, 1, 4, w.n_valid, w.d), generator=g, dtype=torch.int32)
    qkv = qkv.to(torch.int16).view(torch.bfloat16).to(dev)
    spec = dict(kind="all")
    a = lva.VideoBlockSparseAttention(1, 4, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec, device=dev)
    b = lva.VideoBlockSparseAttention(1, 4, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec, device=dev)
    assert a._stacked(qkv[0], qkv[1], qkv[2])
    a.reorder_in(qkv[0], qkv[1], qkv[2])                            # one launch over 3 * B * H planes
    b.reorder_in(qkv[0].clone(), qkv[1].clone(), qkv[2].clone())    # three launches
    torch.cuda.synchronize()
    assert torch.equal(a.qkv_t.view(torch.int16), b.qkv_t.view(torch.int16))
