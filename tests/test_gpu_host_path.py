"""The pinned-host-buffer layer step (copies overlapped with compute per head group) returns
exactly what the device-resident step returns: same kernels on the same rows."""
import numpy as np
import pytest
import torch

from synthetic import WORKLOADS, Workload, make_qkv, mask_variants, spatial_repetition_map, static_calibrated_mask
from tests.gpu_helpers import bits, require_gpu

pytestmark = pytest.mark.gpu


def _run_both(w, spec, static=None, query_src=None, chunks=6, step=3):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    q, k, v = make_qkv(w)
    mk = lambda: lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                               static_mask=static, scale=w.scale, device=dev, query_src=query_src)
    ref_layer = mk()
    o_ref, lse_ref = ref_layer(q.to(dev), k.to(dev), v.to(dev), step=step)
    o_ref, lse_ref = o_ref.cpu(), lse_ref.cpu()
    layer = mk()
    qkvh = torch.stack([q, k, v]).pin_memory()
    oh = torch.full((w.B, w.H, w.n_valid, w.d), float("nan"), dtype=torch.bfloat16).pin_memory()
    lh = torch.full((w.B, w.H, w.n_pad), float("nan"), dtype=torch.float32).pin_memory()
    for _ in range(2):                      # twice: the second call reuses the staging buffers
        layer.forward_host(qkvh, oh, lh, step=step, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        assert lva.lva_device_error() == (0, 0)
        assert np.array_equal(bits(oh), bits(o_ref))
        assert np.array_equal(bits(lh), bits(lse_ref))


def test_host_path_window_mask():
    w = WORKLOADS["small"]
    _run_both(w, mask_variants(w)[0])


def test_host_path_per_head_static_mask_two_batches():
    w = Workload("static_b2", B=2, H=4, d=128, T=3, Hg=16, Wg=32, tile=(1, 8, 16), block_size=128, seed=31)
    _run_both(w, dict(kind="static"), static=static_calibrated_mask(w, 0.4), chunks=5)


def test_host_path_repetitive_heads():
    w = Workload("rep", B=1, H=6, d=128, T=4, Hg=32, Wg=64, tile=(1, 8, 16), block_size=128, seed=32)
    src = spatial_repetition_map(w, repetitive_heads=[1, 4], group_tile_rows=2)
    _run_both(w, dict(kind="window_anchor", unit=w.Hg * w.Wg, radius=1, anchors=2), query_src=src, chunks=3)


def test_host_path_back_to_back_calls_do_not_mix():
    """Four calls without waiting, alternating two inputs, each into its own host buffers:
    the double-buffered device slots must keep every call's data apart."""
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    w = WORKLOADS["small"]
    spec = mask_variants(w)[0]
    inputs = []
    for seed_shift in (0, 1):
        wv = Workload(w.name, B=w.B, H=w.H, d=w.d, T=w.T, Hg=w.Hg, Wg=w.Wg, tile=w.tile,
                      block_size=w.block_size, seed=w.seed + 50 * seed_shift)
        inputs.append(make_qkv(wv))
    ref = []
    for q, k, v in inputs:
        layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                              scale=w.scale, device=dev)
        o, lse = layer(q.to(dev), k.to(dev), v.to(dev), step=7)
        ref.append((o.cpu(), lse.cpu()))
    layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size, spec,
                                          scale=w.scale, device=dev)
    hosts = [torch.stack(list(x)).pin_memory() for x in inputs]
    outs, events = [], []
    for call in range(4):
        oh = torch.full((w.B, w.H, w.n_valid, w.d), float("nan"), dtype=torch.bfloat16).pin_memory()
        lh = torch.full((w.B, w.H, w.n_pad), float("nan"), dtype=torch.float32).pin_memory()
        events.append(layer.forward_host(hosts[call % 2], oh, lh, step=7, wait=False))
        outs.append((oh, lh))
    for call, ev in enumerate(events):
        ev.synchronize()
        oh, lh = outs[call]
        assert np.array_equal(bits(oh), bits(ref[call % 2][0])), call
        assert np.array_equal(bits(lh), bits(ref[call % 2][1])), call
    assert lva.lva_device_error() == (0, 0)
