"""The mask build that allocates nothing (``lva_build_block_mask_noalloc``).

Some callers of this library cannot allocate device memory: a plugin inside a host framework
that owns every device allocation, or a real-time path that may not allocate after start-up.
For them the library keeps the packed static-mask build's scratch in its own 16 MiB device
array.  These tests call that entry point through the C ABI and check that it returns the
same CSR, bit for bit, as the workspace entry point (``lva_build_block_mask_ws``), on calls
in a row that reuse the shared array with different masks, and that a build needing more
than the array holds is refused before anything runs.

This file is named so that pytest collects it last; it needs nothing that other tests set
up, so it passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

from tests.gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu


def _outputs(params, dev):
    import block_sparse_attention_lva_b200 as lva
    nb = params.n_pad // params.block_size
    row_ptr = torch.full((params.mask_heads * nb + 1,), -7, dtype=torch.int32, device=dev)
    col_idx = torch.full((lva.lva_block_mask_max_nnz(params),), -7, dtype=torch.int32, device=dev)
    nnz = torch.full((1,), -7, dtype=torch.int32, device=dev)
    return row_ptr, col_idx, nnz


def _csr(row_ptr, col_idx, nnz):
    torch.cuda.synchronize()
    n = int(nnz.item())
    return row_ptr.cpu().numpy(), col_idx[:n].cpu().numpy(), n


@pytest.mark.parametrize("hm,nb,density", [
    (12, 256, 0.3),     # the static workload's shape (3,072 rows: one-CTA scan)
    (4, 4096, 0.3),     # 16,384 rows of 4,096 blocks: tiled scan, 8.4 MB of the 16 MiB scratch
])
def test_noalloc_build_equals_workspace_build_on_calls_in_a_row(hm, nb, density):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    torch.cuda.set_device(dev)
    p = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 128, nb * 128 - 3, 128, hm)
    assert 0 < lva.lva_block_mask_workspace_bytes(p) <= 16 << 20
    ws = torch.empty(lva.lva_block_mask_workspace_bytes(p), dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev).manual_seed(nb + hm)
    for call in range(2):
        # a different mask on each call, so a stale scratch from the previous call would show
        dense = (torch.rand((hm, nb, nb), generator=g, device=dev) < density * (1 + call)).to(torch.uint8)
        dense[0, call] = 0                                  # an empty row
        dense[-1, -1 - call] = 1                            # a full row
        ref = _outputs(p, dev)
        lva.lva_build_block_mask_ws(p, dense, *ref, ws)
        ref = _csr(*ref)
        got = _outputs(p, dev)
        lva.lva_build_block_mask_noalloc(p, dense, *got)
        got = _csr(*got)
        assert lva.lva_device_error() == (0, 0)
        assert got[2] == ref[2], f"call {call}: nnz {got[2]} != {ref[2]}"
        assert np.array_equal(got[0], ref[0]), f"call {call}: row_ptr differs"
        assert np.array_equal(got[1], ref[1]), f"call {call}: col_idx differs"


def test_noalloc_build_refuses_what_does_not_fit():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    torch.cuda.set_device(dev)
    # 9 heads of 4096 x 4096 blocks need 18.9 MB of scratch: refused on the host, nothing runs
    hm, nb = 9, 4096
    p = lva.MaskParams(lva.LVA_MASK_STATIC, nb * 128, nb * 128, 128, hm)
    assert lva.lva_block_mask_workspace_bytes(p) > 16 << 20
    dense = torch.zeros((hm, nb, nb), dtype=torch.uint8, device=dev)
    row_ptr, col_idx, nnz = _outputs(p, dev)
    with pytest.raises(lva.LvaError, match="LVA_ERR_CAPACITY"):
        lva.lva_build_block_mask_noalloc(p, dense, row_ptr, col_idx, nnz)
    torch.cuda.synchronize()
    assert int(nnz.item()) == -7                           # untouched
