"""The Python binding refuses host tensors before anything reaches the C library: a host
address passed as a device pointer would fault in a kernel (no GPU needed)."""
import pytest
import torch

import block_sparse_attention_lva_b200 as lva


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


B, H, N, NP, D, BS = 1, 2, 250, 256, 64, 64
NB = NP // BS

CALLS = {
    "reorder": lambda: lva.lva_reorder_tokens(_bf16(B * H, N, D), _bf16(B * H, NP, D), (2, 5, 25), (1, 5, 5), NP),
    "build_mask": lambda: lva.lva_build_block_mask(lva.MaskParams(lva.LVA_MASK_ALL, NP, N, BS), None,
                                                   _i32(NB + 1), _i32(NB * NB), _i32(1)),
    "build_mask_static": lambda: lva.lva_build_block_mask(lva.MaskParams(lva.LVA_MASK_STATIC, NP, N, BS),
                                                          torch.ones((1, NB, NB), dtype=torch.uint8),
                                                          _i32(NB + 1), _i32(NB * NB), _i32(1)),
    "attn": lambda: lva.lva_block_sparse_attn(_bf16(B, H, NP, D), _bf16(B, H, NP, D), _bf16(B, H, NP, D),
                                              _bf16(B, H, NP, D), _f32(B, H, NP), N, BS, _i32(NB + 1),
                                              _i32(NB * NB), 1, 0.125),
    "attn_raster": lambda: lva.lva_block_sparse_attn_raster(_bf16(B, H, NP, D), _bf16(B, H, NP, D),
                                                            _bf16(B, H, NP, D), _bf16(B, H, N, D), _f32(B, H, NP),
                                                            N, BS, _i32(NB + 1), _i32(NB * NB), 1, 0.125,
                                                            (2, 5, 25), (1, 5, 5)),
    "window_attn": lambda: lva.lva_window_transposed_attn(_bf16(B, H, 128 * 64, D), _bf16(B, H, 128 * 64, D),
                                                          _bf16(B, H, 128 * 64, D), _bf16(B, H, 128 * 64, D),
                                                          _f32(B, H, 128 * 64), 64, BS, _i32(128 + 1),
                                                          _i32(128 * 128), 1, 0.125),
    "broadcast": lambda: lva.lva_broadcast_blocks(_bf16(B, H, NP, D), _f32(B, H, NP), BS, _i32(1, NB)),
    "energy": lambda: lva.lva_block_energy(_bf16(B, H, NP, D), _bf16(B, H, NP, D), _f32(B, H, NP),
                                           _f32(B, H, NB, NB), N, BS, _i32(NB + 1), _i32(NB * NB), 1, 0.125),
    "select": lambda: lva.lva_select_blocks(_f32(B, H, NB, NB), torch.zeros((B, H, NB, NB), dtype=torch.uint8), 0.9),
    "aggregate": lambda: lva.lva_aggregate_masks(torch.zeros((3, NB * NB), dtype=torch.uint8),
                                                 torch.zeros(NB * NB, dtype=torch.uint8), 0.5),
}


@pytest.mark.parametrize("name", list(CALLS))
def test_host_tensors_are_refused(name):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        CALLS[name]()


class _FakeCudaTensor:
    """Duck-typed stand-in for a CUDA tensor (only what the binding's check reads)."""
    is_cuda = True

    def __init__(self, index):
        self.device = torch.device("cuda", index)
        self.dtype = torch.bfloat16

    def is_contiguous(self):
        return True

    def numel(self):
        return 16


def test_tensors_of_another_device_are_refused(monkeypatch):
    from block_sparse_attention_lva_b200 import _binding
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    _binding._cuda_tensor(_FakeCudaTensor(0), "q", torch.bfloat16, 16)          # current device: accepted
    with pytest.raises(ValueError, match="q is on cuda:1, the current device is cuda:0"):
        _binding._cuda_tensor(_FakeCudaTensor(1), "q", torch.bfloat16, 16)
    with pytest.raises(ValueError, match="q must be torch.float32, got torch.bfloat16"):
        _binding._cuda_tensor(_FakeCudaTensor(0), "q", torch.float32)
    with pytest.raises(ValueError, match="needs 17"):
        _binding._cuda_tensor(_FakeCudaTensor(0), "q", None, 17)
