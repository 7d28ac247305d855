"""Head-sharded layer on one GPU: every rank's shard run in turn gives, for its heads, the
unsharded layer's O and LSE bit for bit (same kernels, same rows; the mask replicated)."""
import numpy as np
import pytest
import torch

from synthetic import WORKLOADS, Workload, make_qkv, mask_variants, spatial_repetition_map, static_calibrated_mask
from tests.gpu_helpers import bits, require_gpu

pytestmark = pytest.mark.gpu


def _check(w, spec, world, static=None, query_src=None, step=0):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    q, k, v = make_qkv(w)
    full = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                         static_mask=static, scale=w.scale, device=dev, query_src=query_src)
    o_ref, lse_ref = (t.cpu() for t in full(q.to(dev), k.to(dev), v.to(dev), step=step))
    for rank in range(world):
        shard = lva.HeadShard(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec, world, rank,
                              static_mask=static, scale=w.scale, device=dev, query_src=query_src)
        h0, h1 = shard.h0, shard.h1
        o, lse = shard(q[:, h0:h1].contiguous().to(dev), k[:, h0:h1].contiguous().to(dev),
                       v[:, h0:h1].contiguous().to(dev), step=step)
        torch.cuda.synchronize()
        assert lva.lva_device_error() == (0, 0)
        assert np.array_equal(bits(o), bits(o_ref[:, h0:h1])), (world, rank)
        assert np.array_equal(bits(lse), bits(lse_ref[:, h0:h1])), (world, rank)


@pytest.mark.parametrize("world", [2, 5])
def test_window_mask_heads_split(world):
    w = WORKLOADS["small"]
    _check(w, mask_variants(w)[0], world, step=9)


@pytest.mark.parametrize("world", [2, 3])
def test_per_head_static_mask_split(world):
    w = WORKLOADS["static"]
    _check(w, dict(kind="static"), world, static=static_calibrated_mask(w))


def test_repetitive_heads_split():
    w = Workload("rep", B=2, H=6, d=128, T=4, Hg=32, Wg=64, tile=(1, 8, 16), block_size=128, seed=33)
    src = spatial_repetition_map(w, repetitive_heads=[1, 4], group_tile_rows=2)
    _check(w, dict(kind="window_anchor", unit=w.Hg * w.Wg, radius=1, anchors=2), 4, query_src=src)
