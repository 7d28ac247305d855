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
