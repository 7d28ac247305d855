"""Workload shapes and seeded input draws for video-DiT-shaped block-sparse attention.

The five workloads mirror the sizes the LVSA, CalibAtt and SQuad pages talk about:
Wan-2.1-like latent grids (21 frames of 30x52 or 45x80 latent tokens, 81 frames for
long video), 12 or 40 heads of dimension 128, 128x128 blocks, and a tiny 256-token case
that a pure-Python check finishes instantly.

Everything here is deterministic from integer seeds, so the same tensors appear on any
machine.  Nothing here computes attention, token order or masks from the method: the
static "calibrated" mask below is a random input (the pages obtain such masks offline
from model calibration, which needs trained weights).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One video-shaped attention problem.

    Tokens of the latent grid ``T x Hg x Wg`` are the sequence; ``tile`` is the 3D tile
    (tt, th, tw) used to reorder them; ``block_size`` is the square attention block.
    """

    name: str
    B: int
    H: int
    d: int
    T: int
    Hg: int
    Wg: int
    tile: tuple
    block_size: int
    seed: int
    k_offset: float = 0.0

    @property
    def n_valid(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def n_pad(self) -> int:
        bs = self.block_size
        return (self.n_valid + bs - 1) // bs * bs

    @property
    def nb(self) -> int:
        return self.n_pad // self.block_size

    @property
    def frame_tokens(self) -> int:
        return self.Hg * self.Wg

    @property
    def scale(self) -> float:
        # float32 value of 1/sqrt(d); both sides use exactly this float.
        return float(np.float32(1.0 / math.sqrt(self.d)))


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, d=64, T=4, Hg=8, Wg=8, tile=(1, 4, 4),
                     block_size=64, seed=0),
    "small": Workload("small", B=1, H=12, d=128, T=21, Hg=30, Wg=52, tile=(1, 8, 16),
                      block_size=128, seed=1),
    "static": Workload("static", B=1, H=12, d=128, T=21, Hg=30, Wg=52, tile=(1, 8, 16),
                       block_size=128, seed=2),
    "large": Workload("large", B=1, H=40, d=128, T=21, Hg=45, Wg=80, tile=(1, 8, 16),
                      block_size=128, seed=3, k_offset=0.5),
    "long": Workload("long", B=1, H=12, d=128, T=81, Hg=30, Wg=52, tile=(1, 8, 16),
                     block_size=128, seed=4),
}


def _head_generator(seed: int, tensor: int, b: int, h: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(((seed * 1_000_003 + tensor * 10_007 + b * 101) * 1009 + h) % (2**62))
    return g


def make_qkv(w: Workload, heads: Optional[Iterable[int]] = None, dtype=torch.bfloat16):
    """Draw raster-order Q, K, V of shape [B, H, n_valid, d] (bf16, round-to-nearest-even).

    Each (tensor, b, h) slice has its own seeded generator, so any subset of heads can be
    drawn alone and matches the full draw.  Values are iid N(0,1) in fp32 before the cast;
    K gets ``w.k_offset`` added to every component (the same vector for all tokens of a
    head) when the workload asks for it.
    """
    hs = list(range(w.H)) if heads is None else list(heads)
    out = []
    for t in range(3):
        x = torch.empty((w.B, len(hs), w.n_valid, w.d), dtype=dtype)
        for b in range(w.B):
            for hi, h in enumerate(hs):
                g = _head_generator(w.seed, t, b, h)
                v = torch.randn((w.n_valid, w.d), generator=g, dtype=torch.float32)
                if t == 1 and w.k_offset != 0.0:
                    v += w.k_offset
                x[b, hi] = v.to(dtype)
        out.append(x)
    return tuple(out)


def make_qk_calibration(w: Workload, prompt: int, heads: Optional[Iterable[int]] = None,
                        strength: float = 9.0, length_scale: float = 0.15,
                        dtype=torch.bfloat16):
    """Raster-order Q, K [B, H, n_valid, d] with space-time locality, one draw per prompt.

    Stand-in for the activations of a video DiT during calibration (which needs trained
    weights): every head has a fixed positional field F_h -- random Fourier features of the
    normalised token position (t/T, y/Hg, x/Wg), F = sqrt(2/d) cos(W p + b) with W ~ N(0,
    1/length_scale^2) and b ~ U[0, 2 pi), seeded by the workload and the head only -- and
    each prompt adds its own N(0, 1) noise:  Q = strength * F + noise_q, K = strength * F +
    noise_k.  <F_r, F_c> approximates exp(-|p_r - p_c|^2 / (2 length_scale^2)), so nearby
    tokens score higher, and the structure is shared by all prompts while the noise is not.
    """
    hs = list(range(w.H)) if heads is None else list(heads)
    t, y, x = torch.meshgrid(torch.arange(w.T), torch.arange(w.Hg), torch.arange(w.Wg), indexing="ij")
    pos = torch.stack([t.reshape(-1) / max(1, w.T), y.reshape(-1) / max(1, w.Hg),
                       x.reshape(-1) / max(1, w.Wg)], dim=1).to(torch.float64)      # [N, 3]
    q = torch.empty((w.B, len(hs), w.n_valid, w.d), dtype=dtype)
    k = torch.empty_like(q)
    for hi, h in enumerate(hs):
        g = _head_generator(w.seed, 7, 0, h)
        freq = torch.randn((3, w.d), generator=g, dtype=torch.float64) / length_scale
        phase = torch.rand((w.d,), generator=g, dtype=torch.float64) * (2 * math.pi)
        field = (math.sqrt(2.0 / w.d) * torch.cos(pos @ freq + phase)).to(torch.float32)
        for b in range(w.B):
            gq = _head_generator(w.seed + 1_000 * (prompt + 1), 8, b, h)
            gk = _head_generator(w.seed + 1_000 * (prompt + 1), 9, b, h)
            q[b, hi] = (strength * field + torch.randn((w.n_valid, w.d), generator=gq)).to(dtype)
            k[b, hi] = (strength * field + torch.randn((w.n_valid, w.d), generator=gk)).to(dtype)
    return q, k


def _block_centroids(w: Workload) -> np.ndarray:
    """Mean latent coordinates (t, y, x) of the real tokens of every block, [nb, 3].

    Tokens are ranked in the spatiotemporal tile order of the workload (tiles of
    ``w.tile`` in raster order of tile coordinates, tokens in raster order inside a tile)
    by one lexicographic sort of their coordinates; this serves only to place the blocks
    of the random mask below and is not part of any computation under test.
    """
    tt, th, tw = w.tile
    t, y, x = np.meshgrid(np.arange(w.T), np.arange(w.Hg), np.arange(w.Wg), indexing="ij")
    t, y, x = t.reshape(-1), y.reshape(-1), x.reshape(-1)
    order = np.lexsort((x % tw, y % th, t % tt, x // tw, y // th, t // tt))
    coords = np.stack([t[order], y[order], x[order]], axis=1).astype(np.float64)
    cent = np.zeros((w.nb, 3))
    for i in range(w.nb):
        blk = coords[i * w.block_size:(i + 1) * w.block_size]
        # a block of padding only sits at the last real token
        cent[i] = blk.mean(axis=0) if len(blk) else coords[-1]
    return cent


def static_calibrated_mask(w: Workload, density: float = 0.30, seed_base: int = 1000) -> np.ndarray:
    """Random per-head static block mask [H, nb, nb] (uint8) standing in for a calibrated mask.

    Block i sits at the centroid (t_i, y_i, x_i) of its real tokens' latent coordinates.
    The spatiotemporal distance of blocks i, j weighs a frame like 8 latent rows or 16
    latent columns (one tile):
        delta_ij = sqrt((t_i - t_j)^2 + ((y_i - y_j) / 8)^2 + ((x_i - x_j) / 16)^2).
    Block (i, j) is kept with probability p_ij = min(1, c * exp(-delta_ij / 2)), and always
    when i == j; c is found by float64 bisection so that the expected density, counting the
    diagonal as 1, equals ``density``.  Head h draws u_ij uniform from numpy's PCG64
    seeded with ``seed_base + h`` and keeps the block when u_ij < p_ij.
    """
    nb = w.nb
    cent = _block_centroids(w)
    dt = cent[:, None, 0] - cent[None, :, 0]
    dy = (cent[:, None, 1] - cent[None, :, 1]) / 8.0
    dx = (cent[:, None, 2] - cent[None, :, 2]) / 16.0
    base = np.exp(-np.sqrt(dt * dt + dy * dy + dx * dx) / 2.0)
    eye = np.eye(nb, dtype=bool)

    def expected(c):
        p = np.minimum(1.0, c * base)
        p[eye] = 1.0
        return p.mean()

    lo, hi = 0.0, 1.0
    while expected(hi) < density:
        hi *= 2.0
    for _ in range(100):
        mid = 0.5 * (lo + hi)
        if expected(mid) < density:
            lo = mid
        else:
            hi = mid
    p = np.minimum(1.0, hi * base)
    masks = np.zeros((w.H, nb, nb), dtype=np.uint8)
    for h in range(w.H):
        draw = np.random.default_rng(seed_base + h).random((nb, nb))
        masks[h] = ((draw < p) | eye).astype(np.uint8)
    return masks


def mask_variants(w: Workload) -> List[dict]:
    """The block-mask specifications each workload is checked and measured with.

    ``window_anchor`` entries give (unit tokens, radius in units, anchors, steps);
    ``static`` entries carry a dense per-head mask; ``two_stage`` gives the window group
    size in blocks; ``all`` is the dense mask; ``lvsa_frames`` gives (frame tokens, global
    frames, frame budget, steps).
    """
    if w.name == "tiny":
        return [dict(label="win1_anchor1", kind="window_anchor", unit=w.block_size, radius=1,
                     anchors=1, steps=[0])]
    if w.name == "small":
        return [dict(label="frame1_anchor4", kind="window_anchor", unit=w.frame_tokens,
                     radius=1, anchors=4, steps=list(range(50)))]
    if w.name == "static":
        return [dict(label="static30", kind="static", density=0.30),
                dict(label="all", kind="all")]
    if w.name == "large":
        return [dict(label=f"band{r}_anchor4", kind="window_anchor", unit=w.block_size,
                     radius=r, anchors=4, steps=[0]) for r in (28, 60, 171)]
    if w.name == "long":
        # Window groups of about sqrt(n) tokens: round(sqrt(n_pad) / Bs) blocks.
        g = int(round(math.sqrt(w.n_pad) / w.block_size))
        return ([dict(label="two_stage", kind="two_stage", group=g)]
                + [dict(label=f"band{r}_anchor4", kind="window_anchor", unit=w.block_size,
                        radius=r, anchors=4, steps=[0]) for r in (23, 48, 130, 287)]
                + [dict(label="all", kind="all")]
                # expanded frame windows: a 21-frame budget (a Wan-2.1-like training horizon)
                # with 4 rotating global frames over the 81 latent frames
                + [dict(label="lvsa_c21_g4", kind="lvsa_frames", unit=w.frame_tokens, anchors=4,
                        budget=21, steps=[0])])
    raise KeyError(w.name)


def spatial_repetition_map(w: Workload, repetitive_heads, group_tile_rows: int) -> np.ndarray:
    """Block source map [H, nb] (int32) for heads whose spatial rows repeat.

    An input, like a calibrated mask: CalibAtt selects repetitive heads offline from the
    similarity of spatial rows, which needs model activations.  Here, in tile order with
    tiles of (1, th, tw) tokens, the tiles of a frame form a grid of tile rows x tile
    columns; for the listed heads every group of ``group_tile_rows`` consecutive tile rows
    takes the output of its first tile row (the anchor), column by column.  A block is
    repeated only when it is one full tile and its anchor tile is full too; every other
    block is computed.  Other heads compute every block.
    """
    tt, th, tw = w.tile
    assert tt == 1 and th * tw == w.block_size
    n_th = (w.Hg + th - 1) // th
    n_tw = (w.Wg + tw - 1) // tw
    # tile sizes and tile-order offsets inside one frame
    offs, sizes = [], []
    pos = 0
    for ih in range(n_th):
        for iw in range(n_tw):
            size = min(th, w.Hg - ih * th) * min(tw, w.Wg - iw * tw)
            offs.append(pos)
            sizes.append(size)
            pos += size
    src = np.tile(np.arange(w.nb, dtype=np.int32), (w.H, 1))
    for t in range(w.T):
        base = t * w.frame_tokens
        for ih in range(n_th):
            a_ih = ih - ih % group_tile_rows
            if a_ih == ih:
                continue
            for iw in range(n_tw):
                me, an = ih * n_tw + iw, a_ih * n_tw + iw
                start, a_start = base + offs[me], base + offs[an]
                if (sizes[me] != w.block_size or sizes[an] != w.block_size
                        or start % w.block_size or a_start % w.block_size):
                    continue
                for h in repetitive_heads:
                    src[h, start // w.block_size] = a_start // w.block_size
    return src
