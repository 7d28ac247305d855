"""Oracle: energy-based block selection and cross-prompt aggregation (test infrastructure only).

CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention"),
section 2 A, the offline calibration phase:

1. energy-based block selection -- the attention matrix is divided into Bs x Bs blocks; for
   every query block, the "energy" toward each key block is the sum of its attention
   scores; the fewest key blocks whose cumulative energy reaches a threshold eps(t) are
   kept (eps is higher early in denoising and lower late);
2. cross-prompt aggregation -- the per-prompt masks are averaged and a block is kept when
   the fraction of calibration prompts that selected it reaches the agreement threshold rho.

The result is a static per-(timestep, layer, head) block mask: the input of the static
mask kind of the CSR builder.

Readings where the page is silent (the plainest form section 2 A supports):

* attention scores are the row-softmax probabilities over all real keys (c < n_valid),
  A[r][c] = exp(s_rc - LSE_r) with s_rc = scale * <q_r, k_c>;
* E[i][j] = sum of A[r][c] over the real rows r of query block i and the real keys c of
  key block j; padded query rows contribute nothing, so a block of padding rows has
  E = 0 everywhere and selects nothing;
* selection order: descending energy, equal energies by ascending key block index; the
  cumulative sums S_k (sum of the first k energies in that order) are taken one addition
  at a time in float64; k = the smallest k >= 0 with S_k >= eps * S_nb, eps in [0, 1];
  a decision taken in float64 on float32 energies, in this exact order, on both sides;
* aggregation: keep a block when count >= rho * P in float64, P = number of prompts.
"""
from __future__ import annotations

import numpy as np

from .attention import _as_f64


def block_energy(q, k, block_size: int, n_valid: int, scale: float, query_blocks=None) -> np.ndarray:
    """Block energies E [B, H, nb, nb] (float64) of dense softmax attention.

    q, k: [B, H, n_pad, d] (bf16-valued); ``scale`` is the caller's float32 value.
    Query block by query block: scores against every real key, the row softmax, then the
    sum of the probabilities inside each key block.  ``query_blocks`` optionally restricts
    the work to a list of (b, h, i) triples; rows not computed are left as NaN.
    """
    q, k = _as_f64(q), _as_f64(k)
    B, H, n_pad, d = q.shape
    bs = block_size
    nb = n_pad // bs
    sc = float(np.float32(scale))
    if query_blocks is None:
        energy = np.zeros((B, H, nb, nb))
        query_blocks = [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    else:
        energy = np.full((B, H, nb, nb), np.nan)
    for b, h, i in query_blocks:
        energy[b, h, i] = 0.0
        keys = k[b, h, :n_valid]
        r0, r1 = i * bs, min((i + 1) * bs, n_valid)
        if r1 <= r0:
            continue                                           # padding rows only
        s = sc * (q[b, h, r0:r1] @ keys.T)                     # [rows, n_valid]
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        a = e / e.sum(axis=1, keepdims=True)                   # row softmax
        for j in range(nb):
            c0, c1 = j * bs, min((j + 1) * bs, n_valid)
            if c1 > c0:
                energy[b, h, i, j] = a[:, c0:c1].sum()
    return energy


def select_row(energy_row, eps: float) -> np.ndarray:
    """Minimal set of key blocks whose cumulative energy reaches eps of the row's total.

    ``energy_row``: 1-D energies (float32 values); returns a bool mask of the same length.
    """
    e = np.asarray(energy_row, dtype=np.float64)
    n = e.shape[0]
    order = sorted(range(n), key=lambda j: (-e[j], j))
    prefix = [0.0]
    for j in order:                                            # one float64 addition at a time
        prefix.append(prefix[-1] + float(e[j]))
    target = float(eps) * prefix[n]
    kcount = n
    for kk in range(n + 1):
        if prefix[kk] >= target:
            kcount = kk
            break
    out = np.zeros(n, dtype=bool)
    for j in order[:kcount]:
        out[j] = True
    return out


def select_blocks(energy, eps: float) -> np.ndarray:
    """``select_row`` applied to every row of the last axis."""
    e = np.asarray(energy)
    flat = e.reshape(-1, e.shape[-1])
    out = np.stack([select_row(row, eps) for row in flat]) if flat.shape[0] else np.zeros(flat.shape, bool)
    return out.reshape(e.shape)


def aggregate_masks(masks, rho: float) -> np.ndarray:
    """Keep a block when at least a fraction rho of the P prompt masks selected it.

    ``masks``: [P, ...] bool/uint8; returns bool [...].
    """
    m = np.asarray(masks).astype(bool)
    p = m.shape[0]
    count = m.sum(axis=0).astype(np.float64)
    return count >= float(rho) * float(p)
