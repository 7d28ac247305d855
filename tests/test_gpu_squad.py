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


@pytest.mark.parametrize("H,n,d,window,bs", [
    (2, 32768, 128, 256, 128),        # m = 128
    (1, 16384, 64, 128, 64),          # m = 128, 64-blocks: a Q box spans two blocks
    (3, 8192, 128, 64, 128),          # m = 128, short windows
])
def test_window_transposed_attn_matches_explicit_transpose(H, n, d, window, bs):
    """Reading the window-transposed rows through 3D tensor maps and storing O back in the
    input order equals transpose -> attention -> inverse transpose, bit for bit; LSE comes
    out in the transposed order.  A random block mask exercises general CSR rows."""
    import block_sparse_attention_lva_b200 as lva
    from oracle.mask import dense_to_csr
    from tests.gpu_helpers import bits
    dev = require_gpu()
    m = n // window
    g = torch.Generator().manual_seed(n + d + window)
    q, k, v = (torch.randn((1, H, n, d), generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
    nb = n // bs
    rng = np.random.default_rng(window)
    masks = rng.random((1, nb, nb)) < 0.3
    masks[0, np.arange(nb), np.arange(nb)] = True
    rp, ci = dense_to_csr(masks)
    row_ptr, col_idx = torch.from_numpy(rp).to(dev), torch.from_numpy(ci).to(dev)
    scale = d ** -0.5
    # explicit: transpose (tile reorder of grid (1, m, w) with tiles (1, m, 1)), attend, invert
    qt, kt, vt = (torch.empty_like(x) for x in (q, k, v))
    for src, dst in ((q, qt), (k, kt), (v, vt)):
        lva.lva_reorder_tokens(src.view(H, n, d), dst.view(H, n, d), (1, m, window), (1, m, 1), n)
    o_t = torch.empty_like(q)
    lse_ref = torch.empty((1, H, n), dtype=torch.float32, device=dev)
    lva.lva_block_sparse_attn(qt, kt, vt, o_t, lse_ref, n, bs, row_ptr, col_idx, 1, scale)
    o_ref = torch.empty_like(q)
    lva.lva_reorder_tokens(o_t.view(H, n, d), o_ref.view(H, n, d), (1, m, window), (1, m, 1), n, inverse=True)
    # fused
    o = torch.full_like(q, float("nan"))
    lse = torch.full((1, H, n), float("nan"), dtype=torch.float32, device=dev)
    lva.lva_window_transposed_attn(q, k, v, o, lse, window, bs, row_ptr, col_idx, 1, scale)
    torch.cuda.synchronize()
    assert lva.lva_device_error() == (0, 0)
    assert np.array_equal(bits(o), bits(o_ref))
    assert np.array_equal(bits(lse), bits(lse_ref))
