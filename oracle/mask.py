"""Oracle: block masks and their per-query-block CSR lists (test infrastructure only).

A block mask M[h_m][i][j] says whether query block i attends key block j (blocks of
``Bs`` tokens in tile order).  Sources:

* Window + rotating anchors -- LVSA page ("LVSA: Training-Free Sparse Attention for Long
  Video Diffusion"), technical summary section 2, "Meccanismo Core": a query frame t
  attends A(t) = G union W(t); W(t) is a local window of frames around t; the global set
  G_s moves by s mod T_per at denoising step s, so that over T_per consecutive steps every
  frame is a global anchor exactly once.
* Static masks -- CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated
  Sparse Attention"), section 2 B "Fase di Inferenza": precomputed per (timestep, layer,
  head) skip lists, no decision at inference time.  The mask is an input and is used as is.
* Two-stage windows -- SQuad page ("SQuad: Sub-Quadratic Attention Distillation for
  Efficient Video Generation"), technical summary section 1: a local pass inside fixed
  windows of size w, and a global pass linking the same relative position across windows;
  w = sqrt(n).

Readings where the pages are silent (the plainest form the passages above support):

* Windows are measured in units of ``U`` tokens (U = H*W gives latent frames when the
  tile depth is 1; U = Bs gives block windows).  Block i spans units lo(i)..hi(i) of its
  real tokens; a block made only of padding takes the unit of the last real token.
  Key block j is in the window of query block i when their unit ranges come within
  ``r`` units of each other.
* Anchors are key blocks, G evenly spaced ones at floor(a*nb/G), all shifted by the step
  s (one block per step), so T_per = nb/G.  Every query block attends every anchor.
* Two-stage: window groups of g consecutive blocks (the last group may be short).  Local
  pass: j in the same group as i.  Global pass: one strided block j = (i + g) mod nb,
  the same relative position in the next group.
* Expanded adaptive windows with frame anchors (LVSA technical summary section 2, "Finestre
  Adattive Espanse" and "Ancore Globali Rotanti"): frames t = 0..T-1 (U tokens each); the
  global frames G_s = {(floor(a*T/G) + s) mod T}; the local window W(t) starts as {t} and
  grows one frame at a time -- right, then left, alternately, continuing on the other side
  at a sequence end -- until |G_s union W(t)| = min(C, T) for the budget C.  A query block
  attends the union of A(t) over the frames its real tokens touch.
"""
from __future__ import annotations

import numpy as np


def window_anchor_mask(n_pad: int, n_valid: int, block_size: int, unit_tokens: int,
                       radius: int, num_anchors: int, step: int) -> np.ndarray:
    """Dense boolean [nb, nb] mask for the local window plus rotating anchors."""
    bs = block_size
    nb = n_pad // bs
    lo = np.empty(nb, dtype=np.int64)
    hi = np.empty(nb, dtype=np.int64)
    last_real_unit = (n_valid - 1) // unit_tokens
    for i in range(nb):
        first = i * bs
        if first >= n_valid:
            lo[i] = hi[i] = last_real_unit
        else:
            last = min((i + 1) * bs, n_valid) - 1
            lo[i] = first // unit_tokens
            hi[i] = last // unit_tokens
    anchors = set()
    for a in range(num_anchors):
        anchors.add((a * nb // num_anchors + step) % nb)
    m = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        for j in range(nb):
            in_window = lo[j] <= hi[i] + radius and hi[j] >= lo[i] - radius
            m[i, j] = in_window or (j in anchors)
    return m


def anchor_set(nb: int, num_anchors: int, step: int) -> set:
    """G_s: the anchor key blocks at denoising step s."""
    return {(a * nb // num_anchors + step) % nb for a in range(num_anchors)}


def two_stage_mask(nb: int, group: int) -> np.ndarray:
    """Dense boolean [nb, nb] mask: local window groups plus one strided cross-group block."""
    m = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        for j in range(nb):
            if j // group == i // group:
                m[i, j] = True
        m[i, (i + group) % nb] = True
    return m


def all_mask(nb: int) -> np.ndarray:
    """The all-ones mask: dense attention."""
    return np.ones((nb, nb), dtype=bool)


def dense_to_csr(masks: np.ndarray):
    """Per-query-block CSR of a stack of masks [H_m, nb, nb].

    Rows are ordered (h_m, i); ``row_ptr`` has H_m*nb + 1 global offsets; each row's
    column indices are ascending and unique.  Returns (row_ptr int32, col_idx int32).
    """
    masks = np.asarray(masks)
    if masks.ndim == 2:
        masks = masks[None]
    hm, nb, nb2 = masks.shape
    assert nb == nb2
    row_ptr = [0]
    cols = []
    for h in range(hm):
        for i in range(nb):
            js = [j for j in range(nb) if masks[h, i, j]]
            cols.extend(js)
            row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int32), np.asarray(cols, dtype=np.int32)


def csr_to_dense(row_ptr: np.ndarray, col_idx: np.ndarray, mask_heads: int, nb: int) -> np.ndarray:
    """Inverse of ``dense_to_csr`` (used to feed a CSR to the attention oracle)."""
    m = np.zeros((mask_heads, nb, nb), dtype=bool)
    for r in range(mask_heads * nb):
        for c in col_idx[row_ptr[r]:row_ptr[r + 1]]:
            m[r // nb, r % nb, c] = True
    return m


def lvsa_frame_sets(num_frames: int, num_anchors: int, step: int, budget: int):
    """A(t) = G_s union W(t) for every frame t, grown frame by frame as described above.

    Returns (anchors, windows, sets): anchors as a set, windows[t] = (lo, hi), sets[t] = A(t).
    """
    T = num_frames
    anchors = {(a * T // num_anchors + step) % T for a in range(num_anchors)} if num_anchors else set()
    target = min(budget, T)
    windows, sets = [], []
    for t in range(T):
        lo = hi = t
        attended = anchors | {t}
        turn_right = True
        while len(attended) < target:
            can_right, can_left = hi + 1 < T, lo - 1 >= 0
            if not (can_right or can_left):
                break
            if (turn_right and can_right) or not can_left:
                hi += 1
                attended.add(hi)
            else:
                lo -= 1
                attended.add(lo)
            turn_right = not turn_right
        windows.append((lo, hi))
        sets.append(attended)
    return anchors, windows, sets


def lvsa_frame_mask(n_pad: int, n_valid: int, block_size: int, frame_tokens: int,
                    num_anchors: int, step: int, budget: int) -> np.ndarray:
    """Dense boolean [nb, nb] block mask of the expanded-window LVSA pattern."""
    bs = block_size
    nb = n_pad // bs
    T = (n_valid + frame_tokens - 1) // frame_tokens
    _, _, sets = lvsa_frame_sets(T, num_anchors, step, budget)

    def frames_of(i):
        first = i * bs
        if first >= n_valid:
            f = (n_valid - 1) // frame_tokens
            return range(f, f + 1)
        last = min((i + 1) * bs, n_valid) - 1
        return range(first // frame_tokens, last // frame_tokens + 1)

    m = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        attended = set()
        for t in frames_of(i):
            attended |= sets[t]
        for j in range(nb):
            m[i, j] = any(f in attended for f in frames_of(j))
    return m
