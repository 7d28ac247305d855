"""Host-side logic of the layer wrapper that needs no GPU."""
import torch

from block_sparse_attention_lva_b200.pipeline import VideoBlockSparseAttention


def test_stacked_detection_needs_one_storage():
    qkv = torch.zeros((3, 1, 2, 16, 8), dtype=torch.bfloat16)
    assert VideoBlockSparseAttention._stacked(qkv[0], qkv[1], qkv[2])
    assert not VideoBlockSparseAttention._stacked(qkv[1], qkv[0], qkv[2])        # out of order
    # separate tensors never count as stacked, whatever their addresses
    q, k, v = (torch.zeros((1, 2, 16, 8), dtype=torch.bfloat16) for _ in range(3))
    assert not VideoBlockSparseAttention._stacked(q, k, v)
    # one storage, right order, but a different shape in the middle
    flat = torch.zeros(3 * 2 * 16 * 8, dtype=torch.bfloat16)
    a, b, c = flat[:256].view(1, 2, 16, 8), flat[256:512].view(1, 2, 16, 8), flat[512:].view(1, 2, 16, 8)
    assert VideoBlockSparseAttention._stacked(a, b, c)
    assert not VideoBlockSparseAttention._stacked(a, b.view(2, 1, 16, 8), c)


def test_layer_rejects_misshapen_static_mask_and_query_src():
    import pytest
    # grid 2x8x8 = 128 tokens in 64-token blocks: nb = 2
    kw = dict(B=1, H=3, d=64, grid=(2, 8, 8), tile=(1, 4, 4), block_size=64, device="cpu")
    with pytest.raises(ValueError, match="static_mask"):
        VideoBlockSparseAttention(mask={"kind": "static"}, static_mask=torch.ones(2, 2, 2, dtype=torch.uint8), **kw)
    with pytest.raises(ValueError, match="static_mask"):
        VideoBlockSparseAttention(mask={"kind": "static"}, static_mask=torch.ones(3, 2, 3, dtype=torch.uint8), **kw)
    with pytest.raises(ValueError, match="static_mask"):
        VideoBlockSparseAttention(mask={"kind": "static"}, static_mask=torch.ones(12, dtype=torch.uint8), **kw)
    layer = VideoBlockSparseAttention(mask={"kind": "static"}, static_mask=torch.ones(3, 2, 2, dtype=torch.uint8), **kw)
    assert layer.mask_heads == 3
    win = {"kind": "window_anchor", "unit": 64, "radius": 1, "anchors": 0}
    with pytest.raises(ValueError, match="query_src"):
        VideoBlockSparseAttention(mask=win, query_src=torch.zeros(2, 2, dtype=torch.int32), **kw)
    with pytest.raises(ValueError, match="query_src"):
        VideoBlockSparseAttention(mask=win, query_src=torch.zeros(1, 3, dtype=torch.int32), **kw)
    VideoBlockSparseAttention(mask=win, query_src=torch.zeros(1, 2, dtype=torch.int32), **kw)


def test_host_step_rejects_bad_buffers_before_any_copy():
    import pytest
    kw = dict(B=1, H=2, d=64, grid=(2, 8, 8), tile=(1, 4, 4), block_size=64, device="cpu")
    layer = VideoBlockSparseAttention(mask={"kind": "all"}, **kw)
    N, n_pad = 128, 128
    qkv = torch.zeros((3, 1, 2, N, 64), dtype=torch.bfloat16)
    o = torch.zeros((1, 2, N, 64), dtype=torch.bfloat16)
    lse = torch.zeros((1, 2, n_pad), dtype=torch.float32)
    with pytest.raises(ValueError, match="qkv_host"):
        layer.forward_host(qkv[:, :, :1], o, lse)                        # wrong head count
    with pytest.raises(ValueError, match="o_host"):
        layer.forward_host(qkv, o.float(), lse)                          # wrong dtype
    with pytest.raises(ValueError, match="lse_host"):
        layer.forward_host(qkv, o, torch.zeros((1, 2, n_pad, 2))[..., 0])  # not contiguous
    with pytest.raises(ValueError, match="pinned"):
        layer.forward_host(qkv, o, lse)                                  # pageable host memory
    assert not hasattr(layer, "_host_io")                                # nothing was allocated
