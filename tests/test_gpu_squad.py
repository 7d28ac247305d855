"""SQuad's two-stage operator through the C ABI vs the FP64 oracle."""
import numpy as np
import pytest
import torch

from oracle.attention import squad_two_pass
from tests.gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,n,d,window,stacked", [
    (2, 32768, 128, 256, True),       # m = 128
    (2, 16384, 128, 128, False),      # w = m = 128
    (1, 65536, 64, 512, True),        # d = 64, m = 128
])
def test_squad_matches_oracle(H, n, d, window, stacked):
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    g = torch.Generator().manual_seed(n + window)
    qkv = torch.randn((3, 1, H, n, d), generator=g).to(torch.bfloat16)
    op = lva.SquadTwoPass(1, H, n, d, window, device=dev)
    qd = qkv.to(dev)
    if stacked:
        o = op(qd[0], qd[1], qd[2])
    else:
        o = op(qd[0].clone(), qd[1].clone(), qd[2].clone())
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    ref, ref_local = squad_two_pass(qkv[0], qkv[1], qkv[2], window, op.scale)
    dl = np.abs(op.o_local.float().cpu().numpy() - ref_local)
    assert dl.max() <= 1e-2 and dl.mean() <= 1e-3
    err = np.abs(o.float().cpu().numpy() - ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())


def test_window_transpose_roundtrip_groups_positions():
    # The reorder with grid (1, m, w) and tiles (1, m, 1) puts position p of every window
    # together: token a*w + p lands at p*m + a.
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    n, w = 32768, 256
    m = n // w
    iota = torch.arange(n, dtype=torch.int32, device=dev).view(1, n, 1).view(torch.float32)
    out = torch.empty_like(iota)
    lva.lva_reorder_tokens(iota, out, (1, m, w), (1, m, 1), n)
    got = out.view(torch.int32).cpu().numpy().ravel()
    a, p = np.divmod(got, w)
    assert np.array_equal(p * m + a, np.arange(n))
