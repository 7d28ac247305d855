"""Oracle: block-masked softmax attention in float64 (test infrastructure only).

What is computed: softmax self-attention where query row r (in query block i) attends
only the keys of key blocks j with M[i][j] set -- the block-sparse attention of the LVSA
page ("LVSA: Training-Free Sparse Attention for Long Video Diffusion", technical summary
section 2: attention restricted to A(t) through a block-sparse mechanism) and of the
CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention",
section 2 B: attention only on the selected blocks of the skip list).  With the all-ones
mask it is ordinary dense softmax attention.

Readings (the pages give no formula beyond standard softmax attention):

* scores s_c = scale * <q_r, k_c>, with ``scale`` the caller's float32 value taken exactly;
* keys c >= n_valid (sequence padding) are never attended;
* O_r = sum_c exp(s_c - m) v_c / sum_c exp(s_c - m),  LSE_r = m + ln(sum_c exp(s_c - m))
  with m = max_c s_c (natural logarithm, scale included);
* a row with no attended key has O_r = 0 and LSE_r = -inf;
* padded query rows (r >= n_valid) are computed like any other row.

Inputs arrive as bf16-valued arrays; they are widened to float64 exactly.
"""
from __future__ import annotations

import numpy as np


def _as_f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def attention_blocked(q, k, v, masks, block_size: int, n_valid: int, scale: float,
                      query_blocks=None, return_probs: bool = False):
    """Block-masked attention, one query block at a time.

    q, k, v: [B, H, n_pad, d]; masks: bool [H_m, nb, nb] with H_m in {1, H} (H_m == 1 is
    broadcast to every head).  ``query_blocks`` optionally restricts the work to a list of
    (b, h, i) triples; rows not computed are left as NaN.  Returns (O, LSE) as float64
    arrays [B, H, n_pad, d] and [B, H, n_pad] (plus P per (b, h, i) if ``return_probs``).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    masks = np.asarray(masks, dtype=bool)
    if masks.ndim == 2:
        masks = masks[None]
    B, H, n_pad, d = q.shape
    bs = block_size
    nb = n_pad // bs
    hm = masks.shape[0]
    assert hm in (1, H) and masks.shape[1:] == (nb, nb)
    sc = float(np.float32(scale))

    out = np.full((B, H, n_pad, d), np.nan)
    lse = np.full((B, H, n_pad), np.nan)
    probs = {}
    if query_blocks is None:
        query_blocks = [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    for b, h, i in query_blocks:
        mask_row = masks[h if hm == H else 0, i]
        keys = np.concatenate([np.arange(j * bs, (j + 1) * bs) for j in range(nb) if mask_row[j]]
                              + [np.zeros(0, dtype=np.int64)])
        keys = keys[keys < n_valid]
        rows = slice(i * bs, (i + 1) * bs)
        if keys.size == 0:
            out[b, h, rows] = 0.0
            lse[b, h, rows] = -np.inf
            continue
        s = sc * (q[b, h, rows] @ k[b, h, keys].T)           # [bs, |J|]
        m = s.max(axis=1, keepdims=True)                     # first pass: row max
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)                     # second pass: row sum
        out[b, h, rows] = (e @ v[b, h, keys]) / l
        lse[b, h, rows] = (m + np.log(l))[:, 0]
        if return_probs:
            probs[(b, h, i)] = (keys, e / l)
    if return_probs:
        return out, lse, probs
    return out, lse


def attention_bruteforce(q, k, v, masks, block_size: int, n_valid: int, scale: float):
    """Same operator through an explicit token-level mask and a full softmax (tiny sizes).

    E[r][c] = M[r // Bs][c // Bs] and c < n_valid; masked scores are -inf.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    masks = np.asarray(masks, dtype=bool)
    if masks.ndim == 2:
        masks = masks[None]
    B, H, n_pad, d = q.shape
    bs = block_size
    hm = masks.shape[0]
    sc = float(np.float32(scale))
    cols = np.arange(n_pad)
    out = np.zeros((B, H, n_pad, d))
    lse = np.zeros((B, H, n_pad))
    for b in range(B):
        for h in range(H):
            m = masks[h if hm == H else 0]
            elem = m[np.arange(n_pad)[:, None] // bs, cols[None, :] // bs] & (cols[None, :] < n_valid)
            s = np.where(elem, sc * (q[b, h] @ k[b, h].T), -np.inf)
            for r in range(n_pad):
                if not elem[r].any():
                    out[b, h, r] = 0.0
                    lse[b, h, r] = -np.inf
                    continue
                mx = s[r].max()
                w = np.exp(s[r] - mx)
                out[b, h, r] = (w / w.sum()) @ v[b, h]
                lse[b, h, r] = mx + np.log(w.sum())
    return out, lse


def attention_with_broadcast(q, k, v, masks, block_size: int, n_valid: int, scale: float, query_src):
    """Repetitive heads: only anchor query blocks are computed, the others copy an anchor.

    CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention"),
    section 2 A.3 and B: for a head marked repetitive, attention is computed for a subset of
    rows (the anchors) and the result is replicated to the other rows.  Reading (block
    granularity, tile order): ``query_src`` [S, nb] (S in {1, H}) names for every query block
    i the block whose O rows and LSE it takes; query_src[h][i] == i marks a computed block,
    and every source must itself be computed.
    """
    q_, k_, v_ = _as_f64(q), _as_f64(k), _as_f64(v)
    src = np.asarray(query_src)
    if src.ndim == 1:
        src = src[None]
    B, H, n_pad, d = q_.shape
    nb = n_pad // block_size
    blocks = [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)
              if src[h if src.shape[0] == H else 0, i] == i]
    out, lse = attention_blocked(q, k, v, masks, block_size, n_valid, scale, query_blocks=blocks)
    for b in range(B):
        for h in range(H):
            row = src[h if src.shape[0] == H else 0]
            for i in range(nb):
                j = int(row[i])
                if j != i:
                    assert row[j] == j, "a source block must be computed"
                    out[b, h, i * block_size:(i + 1) * block_size] = out[b, h, j * block_size:(j + 1) * block_size]
                    lse[b, h, i * block_size:(i + 1) * block_size] = lse[b, h, j * block_size:(j + 1) * block_size]
    return out, lse


def squad_two_pass(q, k, v, window: int, scale: float):
    """SQuad's two-stage operator, token by token, in float64.

    SQuad page ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video
    Generation"), technical summary section 1: a local pass mixes tokens inside fixed windows
    of w tokens; a global pass mixes the tokens at the same relative position in every
    window; the local output is the value stream of the global pass.  Reading: both passes
    use the same Q and K; token k = a*w + p sits at position p of window a (n = m*w tokens).

      O_L[a*w + p] = softmax_{p'} (scale q_{a*w+p} . k_{a*w+p'}) v_{a*w+p'}
      O[a*w + p]   = softmax_{a'} (scale q_{a*w+p} . k_{a'*w+p}) O_L[a'*w+p]
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, n, d = q.shape
    assert n % window == 0
    m = n // window
    sc = float(np.float32(scale))
    o_local = np.empty_like(v)
    out = np.empty_like(v)
    for b in range(B):
        for h in range(H):
            for a in range(m):
                idx = np.arange(a * window, (a + 1) * window)
                s = sc * (q[b, h, idx] @ k[b, h, idx].T)
                e = np.exp(s - s.max(axis=1, keepdims=True))
                o_local[b, h, idx] = (e / e.sum(axis=1, keepdims=True)) @ v[b, h, idx]
            for p in range(window):
                idx = np.arange(p, n, window)
                s = sc * (q[b, h, idx] @ k[b, h, idx].T)
                e = np.exp(s - s.max(axis=1, keepdims=True))
                out[b, h, idx] = (e / e.sum(axis=1, keepdims=True)) @ o_local[b, h, idx]
    return out, o_local
