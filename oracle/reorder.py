"""Oracle: the spatiotemporal-tile token order (test infrastructure only).

Why tiles: the LVSA page ("LVSA: Training-Free Sparse Attention for Long Video
Diffusion", technical summary, section 2 "Meccanismo Core") restricts each query frame to
a set of frames, and the CalibAtt page ("Accelerating Text-to-Video Generation with
Calibrated Sparse Attention", section 2, step A.1) works on 128x128 blocks of the attention
matrix.  Blocks only line up with spatiotemporal neighbourhoods when the sequence is
ordered tile by tile.  The pages do not spell the order out; the reading used here is:

* tiles of ``tt x th x tw`` tokens, enumerated raster order (t-tile, then h-tile, then
  w-tile);
* inside a tile, tokens in raster order (t, then h, then w);
* tiles at the grid's far edges are partial (tokens outside the grid are skipped, not
  padded); padding exists only at the end of the sequence.
"""
from __future__ import annotations

import numpy as np


def tile_permutation(T: int, H: int, W: int, tt: int, th: int, tw: int) -> np.ndarray:
    """perm[k] = raster index t*H*W + h*W + w of the k-th token in tile order.

    Built by walking tiles and the tokens inside each tile with plain nested loops.
    """
    perm = []
    for t0 in range(0, T, tt):
        for h0 in range(0, H, th):
            for w0 in range(0, W, tw):
                for t in range(t0, min(t0 + tt, T)):
                    for h in range(h0, min(h0 + th, H)):
                        for w in range(w0, min(w0 + tw, W)):
                            perm.append(t * H * W + h * W + w)
    return np.asarray(perm, dtype=np.int64)


def reorder_forward(src: np.ndarray, perm: np.ndarray, n_pad: int) -> np.ndarray:
    """Gather raster rows into tile order: dst[p, k] = src[p, perm[k]] for k < N.

    ``src`` is [planes, N, row...]; rows N..n_pad-1 of the result are zero.
    """
    n = perm.shape[0]
    assert src.shape[1] == n and n_pad >= n
    dst = np.zeros((src.shape[0], n_pad) + src.shape[2:], dtype=src.dtype)
    for k in range(n):
        dst[:, k] = src[:, perm[k]]
    return dst


def reorder_inverse(src: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Scatter tile-order rows back to raster order: dst[p, perm[k]] = src[p, k], k < N.

    Pad rows (k >= N) of ``src`` are dropped.
    """
    n = perm.shape[0]
    dst = np.zeros((src.shape[0], n) + src.shape[2:], dtype=src.dtype)
    for k in range(n):
        dst[:, perm[k]] = src[:, k]
    return dst
