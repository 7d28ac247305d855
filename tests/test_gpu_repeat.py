"""Repetitive heads (anchor blocks computed, the rest broadcast) vs the FP64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle.attention import attention_with_broadcast
from oracle.mask import dense_to_csr, window_anchor_mask
from synthetic import Workload, make_qkv, spatial_repetition_map
from tests.gpu_helpers import check_o_lse, require_gpu

pytestmark = pytest.mark.gpu

# Frames of 32 x 64 latent tokens: 16 tiles of 8 x 16 = 16 whole 128-token blocks per frame.
ALIGNED = Workload("aligned", B=1, H=4, d=128, T=6, Hg=32, Wg=64, tile=(1, 8, 16), block_size=128, seed=11)


def _gpu(w, masks, src):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    q, k, v = (torch.randn((w.B, w.H, w.n_pad, w.d), generator=torch.Generator().manual_seed(s)).to(torch.bfloat16)
               for s in (1, 2, 3))
    rp, ci = dense_to_csr(masks)
    o = torch.full((w.B, w.H, w.n_pad, w.d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((w.B, w.H, w.n_pad), float("nan"), dtype=torch.float32, device=dev)
    qs = torch.from_numpy(src).to(dev)
    lva.lva_block_sparse_attn(q.to(dev), k.to(dev), v.to(dev), o, lse, w.n_valid, w.block_size,
                              torch.from_numpy(rp).to(dev), torch.from_numpy(ci).to(dev), masks.shape[0],
                              w.scale, query_src=qs)
    lva.lva_broadcast_blocks(o, lse, w.block_size, qs)
    torch.cuda.synchronize()
    return q, k, v, o, lse, lva.lva_device_error()


@pytest.mark.parametrize("heads,group", [((0, 2), 2), ((1,), 4), ((0, 1, 2, 3), 3)])
def test_repetitive_heads_match_oracle(heads, group):
    w = ALIGNED
    src = spatial_repetition_map(w, heads, group)
    assert (src != np.arange(w.nb)).sum() > 0
    m = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, w.frame_tokens, 1, 2, 0)[None]
    q, k, v, o, lse, st = _gpu(w, m, src)
    assert st == (0, 0)
    o_ref, lse_ref = attention_with_broadcast(q, k, v, m, w.block_size, w.n_valid, w.scale, src)
    check_o_lse(o, lse, o_ref, lse_ref, f"repeat {heads} g{group}")


def test_shared_map_and_non_anchor_source_reported():
    w = ALIGNED
    src = spatial_repetition_map(w, (0,), 2)[:1].copy()            # one map for all heads
    m = np.ones((1, w.nb, w.nb), bool)
    q, k, v, o, lse, st = _gpu(w, m, src)
    assert st == (0, 0)
    o_ref, lse_ref = attention_with_broadcast(q, k, v, m, w.block_size, w.n_valid, w.scale, src)
    check_o_lse(o, lse, o_ref, lse_ref, "shared map")
    # a chain (source that is not an anchor) is reported and skipped, never followed
    bad = src.copy()
    i = int(np.flatnonzero(bad[0] != np.arange(w.nb))[0])
    j = int(np.flatnonzero(bad[0] != np.arange(w.nb))[1])
    bad[0, i] = j
    _, _, _, o2, lse2, st2 = _gpu(w, m, bad)
    assert st2[0] == 1 and st2[1] == i


def test_layer_path_with_repetitive_heads():
    import block_sparse_attention_lva_b200 as lva
    from oracle.reorder import reorder_forward, tile_permutation
    dev = require_gpu()
    w = ALIGNED
    src = spatial_repetition_map(w, (1, 3), 2)
    spec = dict(kind="window_anchor", unit=w.frame_tokens, radius=1, anchors=2)
    q, k, v = make_qkv(w)
    layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                          scale=w.scale, device=dev, query_src=src)
    layer(q.to(dev), k.to(dev), v.to(dev), step=0)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    perm = tile_permutation(w.T, w.Hg, w.Wg, *w.tile)
    P = w.B * w.H
    tq, tk, tv = (torch.from_numpy(reorder_forward(x.view(torch.int16).reshape(P, w.n_valid, w.d).numpy(), perm,
                                                   w.n_pad)).view(torch.bfloat16).reshape(w.B, w.H, w.n_pad, w.d)
                  for x in (q, k, v))
    m = window_anchor_mask(w.n_pad, w.n_valid, w.block_size, w.frame_tokens, 1, 2, 0)[None]
    o_ref, lse_ref = attention_with_broadcast(tq, tk, tv, m, w.block_size, w.n_valid, w.scale, src)
    check_o_lse(layer.o_t, layer.lse, o_ref, lse_ref, "layer path")
