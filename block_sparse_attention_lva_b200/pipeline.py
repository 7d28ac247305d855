"""One attention layer's hot path over the C ABI: tile reorder -> CSR -> attention -> inverse.

``VideoBlockSparseAttention`` owns the device buffers of a fixed problem shape (allocated
once through torch, which is used only for device memory and streams) and runs, per call:

1. ``lva_reorder_tokens`` on Q, K and V (raster [B, H, N, d] -> tile order [B, H, n_pad, d]);
2. ``lva_build_block_mask`` for the current denoising step (window + rotating anchors
   change with the step; static, two-stage and all-ones masks are built once);
3. ``lva_block_sparse_attn`` -> O (tile order) and LSE;
4. ``lva_reorder_tokens`` inverse on O (tile order -> raster [B, H, N, d]).

Steps 3 and 4 run as one launch (``lva_block_sparse_attn_raster``) unless repetitive heads
need the tile-order broadcast between them.
"""
from __future__ import annotations

import ctypes

import torch

from . import _binding as lb


def mask_params_for(spec: dict, n_pad: int, n_valid: int, block_size: int, mask_heads: int = 1,
                    step: int = 0) -> lb.MaskParams:
    """``MaskParams`` for a mask specification dict (kind, unit, radius, anchors, group)."""
    kind = spec["kind"]
    if kind == "window_anchor":
        return lb.MaskParams(lb.LVA_MASK_WINDOW_ANCHOR, n_pad, n_valid, block_size, 1,
                             spec["unit"], spec["radius"], spec["anchors"], step)
    if kind == "two_stage":
        return lb.MaskParams(lb.LVA_MASK_TWO_STAGE, n_pad, n_valid, block_size, 1, group_blocks=spec["group"])
    if kind == "all":
        return lb.MaskParams(lb.LVA_MASK_ALL, n_pad, n_valid, block_size, 1)
    if kind == "lvsa_frames":
        return lb.MaskParams(lb.LVA_MASK_LVSA_FRAMES, n_pad, n_valid, block_size, 1, spec["unit"],
                             num_anchors=spec["anchors"], step=step, budget_frames=spec["budget"])
    if kind == "static":
        return lb.MaskParams(lb.LVA_MASK_STATIC, n_pad, n_valid, block_size, mask_heads)
    raise ValueError(f"unknown mask kind {kind!r}")


class VideoBlockSparseAttention:
    """Block-sparse self-attention over a T x Hg x Wg latent video grid.

    ``mask`` is a specification dict; for ``kind == "static"`` pass the dense per-head block
    mask (uint8 [H_m, nb, nb], any device) as ``static_mask``.  ``query_src`` ([1 or H, nb]
    int32) marks repetitive heads: their non-anchor query blocks are not computed and take
    the output of the anchor block they name.
    """

    def __init__(self, B, H, d, grid, tile, block_size, mask: dict, static_mask=None,
                 scale=None, device="cuda", query_src=None):
        self.B, self.H, self.d = B, H, d
        self.grid, self.tile, self.block_size = tuple(grid), tuple(tile), block_size
        self.n_valid = grid[0] * grid[1] * grid[2]
        self.n_pad = (self.n_valid + block_size - 1) // block_size * block_size
        self.nb = self.n_pad // block_size
        self.mask = dict(mask)
        self.scale = float(scale) if scale is not None else float(torch.tensor(d ** -0.5, dtype=torch.float32))
        self.device = torch.device(device)
        self.mask_heads = 1
        self.dense_mask = None
        if mask["kind"] == "static":
            if static_mask is None:
                raise ValueError("static mask kind needs static_mask")
            sm = torch.as_tensor(static_mask, dtype=torch.uint8)
            if sm.dim() != 3 or sm.shape[0] not in (1, H) or tuple(sm.shape[1:]) != (self.nb, self.nb):
                raise ValueError(f"static_mask must have shape [1 or {H}, {self.nb}, {self.nb}], "
                                 f"got {tuple(sm.shape)}")
            self.mask_heads = sm.shape[0]
            self.dense_mask = sm.to(self.device).contiguous()
        self.params = mask_params_for(self.mask, self.n_pad, self.n_valid, block_size, self.mask_heads)
        cap = lb.lva_block_mask_max_nnz(self.params)
        if cap <= 0:
            raise ValueError(f"invalid mask parameters {self.params}")
        kw = dict(device=self.device)
        shape = (B, H, self.n_pad, d)
        # Q, K, V in tile order share one buffer so that a stacked raster QKV is reordered
        # by a single launch.
        self.qkv_t = torch.empty((3,) + shape, dtype=torch.bfloat16, **kw)
        self.q_t, self.k_t, self.v_t = self.qkv_t[0], self.qkv_t[1], self.qkv_t[2]
        self.o_t = torch.empty(shape, dtype=torch.bfloat16, **kw)
        self.lse = torch.empty((B, H, self.n_pad), dtype=torch.float32, **kw)
        self.o = torch.empty((B, H, self.n_valid, d), dtype=torch.bfloat16, **kw)
        self.row_ptr = torch.empty(self.mask_heads * self.nb + 1, dtype=torch.int32, **kw)
        self.col_idx = torch.empty(cap, dtype=torch.int32, **kw)
        self.nnz = torch.empty(1, dtype=torch.int32, **kw)
        # Static masks are built through the workspace path (the dense mask read once).
        ws = lb.lva_block_mask_workspace_bytes(self.params)
        self.mask_ws = torch.empty(ws, dtype=torch.uint8, **kw) if ws > 0 else None
        self.query_src = (torch.as_tensor(query_src, dtype=torch.int32).to(self.device).contiguous()
                          if query_src is not None else None)
        if self.query_src is not None and (self.query_src.dim() != 2 or self.query_src.shape[0] not in (1, H)
                                           or self.query_src.shape[1] != self.nb):
            raise ValueError(f"query_src must have shape [1 or {H}, {self.nb}]")
        self._built_step = None
        self.col_view = self.col_idx

    def build_mask(self, step: int = 0):
        """(Re)build the CSR; parametric window masks depend on the denoising step."""
        steps_matter = self.mask["kind"] in ("window_anchor", "lvsa_frames") and self.mask.get("anchors", 0) > 0
        key = step if steps_matter else 0
        if self._built_step == key:
            return
        self.params.step = key
        lb.lva_build_block_mask_ws(self.params, self.dense_mask, self.row_ptr, self.col_idx, self.nnz,
                                   self.mask_ws)
        self._built_step = key
        # A mask built once can tell the attention call its exact entry count (read back once);
        # short rows then get CTAs that walk several query blocks.  Per-step masks keep the
        # capacity, so no step waits for a device-to-host read.
        self.col_view = self.col_idx
        if not steps_matter:
            self.col_view = self.col_idx[:max(1, int(self.nnz.item()))]

    @staticmethod
    def _stacked(q, k, v):
        """True when q, k, v are consecutive, equally sized, contiguous slices of one buffer.

        Adjacent addresses are not enough: three separate allocations can sit back to back,
        and a view spanning them would leave the first tensor's storage.
        """
        if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
            return False
        sq = q.untyped_storage()
        if not (sq.data_ptr() == k.untyped_storage().data_ptr() == v.untyped_storage().data_ptr()):
            return False
        nbytes = q.numel() * q.element_size()
        return (k.data_ptr() == q.data_ptr() + nbytes and v.data_ptr() == k.data_ptr() + nbytes
                and q.shape == k.shape == v.shape and q.dtype == k.dtype == v.dtype)

    def reorder_in(self, q, k, v):
        P = self.B * self.H
        if self._stacked(q, k, v):
            base = q.view(-1)
            src = torch.as_strided(base, (3 * P, self.n_valid, self.d), (self.n_valid * self.d, self.d, 1))
            lb.lva_reorder_tokens(src, self.qkv_t.view(3 * P, self.n_pad, self.d), self.grid, self.tile,
                                  self.n_pad, inverse=False)
            return
        for src, dst in ((q, self.q_t), (k, self.k_t), (v, self.v_t)):
            lb.lva_reorder_tokens(src.view(P, self.n_valid, self.d), dst.view(P, self.n_pad, self.d),
                                  self.grid, self.tile, self.n_pad, inverse=False)

    def attend(self):
        lb.lva_block_sparse_attn(self.q_t, self.k_t, self.v_t, self.o_t, self.lse, self.n_valid,
                                 self.block_size, self.row_ptr, self.col_view, self.mask_heads, self.scale,
                                 self.query_src)
        if self.query_src is not None:
            lb.lva_broadcast_blocks(self.o_t, self.lse, self.block_size, self.query_src)

    def attend_to_raster(self):
        """Attention with the inverse reorder fused into its epilogue: O goes straight to
        raster order (``self.o``); LSE stays in tile order (``self.lse``)."""
        lb.lva_block_sparse_attn_raster(self.q_t, self.k_t, self.v_t, self.o, self.lse, self.n_valid,
                                        self.block_size, self.row_ptr, self.col_view, self.mask_heads,
                                        self.scale, self.grid, self.tile)

    def reorder_out(self):
        P = self.B * self.H
        lb.lva_reorder_tokens(self.o_t.view(P, self.n_pad, self.d), self.o.view(P, self.n_valid, self.d),
                              self.grid, self.tile, self.n_pad, inverse=True)

    def __call__(self, q, k, v, step: int = 0):
        """Raster-order bf16 Q, K, V [B, H, N, d] on this device -> raster O (the internal
        buffer ``self.o``) and tile-order LSE ``self.lse``."""
        self.reorder_in(q, k, v)
        self.build_mask(step)
        if self.query_src is None:
            self.attend_to_raster()        # steps 3 and 4 in one launch
        else:
            self.attend()                  # repetitive heads broadcast in tile order
            self.reorder_out()
        return self.o, self.lse


    def forward_host(self, qkv_host, o_host, lse_host, step: int = 0, chunks: int = 6, wait: bool = True):
        """One layer step from and to pinned host memory, through ``lva_layer_step_host``.

        ``qkv_host``: pinned bf16 [3, B, H, N, d] (raster Q, K, V); ``o_host``: pinned bf16
        [B, H, N, d] (raster O, written); ``lse_host``: pinned fp32 [B, H, n_pad] (tile-order
        LSE, written).  The C call runs the step per group of heads (about ``chunks`` groups),
        with each group's host-to-device copy, compute and device-to-host copy on three
        streams, so one group's copies overlap the others' compute.  Two device buffer sets
        (staging, outputs, events) are used alternately, so consecutive calls overlap as well.

        Returns a CUDA event that completes when ``o_host`` and ``lse_host`` hold this step's
        results; the host buffers must not be rewritten or read before then.  With ``wait``
        the caller's current stream is also ordered after it (synchronise that stream before
        reading the results on the host).
        """
        B, H, N, d = self.B, self.H, self.n_valid, self.d
        bufs = (("qkv_host", qkv_host, (3, B, H, N, d), torch.bfloat16),
                ("o_host", o_host, (B, H, N, d), torch.bfloat16),
                ("lse_host", lse_host, (B, H, self.n_pad), torch.float32))
        for name, t, shape, dtype in bufs:
            if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {shape}")
        for name, t, _, _ in bufs:
            if not t.is_pinned():
                raise ValueError(f"{name} must be in pinned host memory (copies overlap compute)")
        cur = torch.cuda.current_stream(self.device)
        if not hasattr(self, "_host_io"):
            mk = lambda shape, dt: torch.empty(shape, dtype=dt, device=self.device)
            groups = B * -(-H // -(-H // max(1, min(H, -(-chunks // B)))))
            sets = []
            for _ in range(2):
                events = [torch.cuda.Event() for _ in range(2 * groups + 2)]
                for ev in events:                 # creates the CUDA events (a no-op on the stream)
                    ev.record(cur)
                arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
                t = dict(qkv=mk((3, B, H, N, d), torch.bfloat16), o=mk((B, H, N, d), torch.bfloat16),
                         lse=mk((B, H, self.n_pad), torch.float32), events=events, arr=arr)
                t["c"] = lb.LvaHostStepBuffers(
                    t["qkv"].data_ptr(), t["o"].data_ptr(), t["lse"].data_ptr(), self.qkv_t.data_ptr(),
                    self.o_t.data_ptr(), self.row_ptr.data_ptr(), self.col_idx.data_ptr(), self.col_idx.numel(),
                    self.col_idx.numel(), self.nnz.data_ptr(), arr, len(events))
                sets.append(t)
            self._host_io = dict(sets=sets, slot=0, chunks=chunks,
                                 h2d=torch.cuda.Stream(self.device), d2h=torch.cuda.Stream(self.device),
                                 shape=lb.LvaLayerShape(B, H, d, self.block_size, *self.grid, *self.tile, self.scale))
        io = self._host_io
        if chunks != io["chunks"]:
            raise ValueError(f"chunks is fixed at the first call ({io['chunks']})")
        t = io["sets"][io["slot"]]
        io["slot"] ^= 1
        # The CSR for this step (built on the current stream, which also runs the step's
        # compute); the C call then uses it as it stands.
        self.build_mask(step)
        t["c"].col_len = self.col_view.numel()
        done = lb.lva_layer_step_host(qkv_host, o_host, lse_host, io["shape"], self.params, self.dense_mask,
                                      False, self.query_src, t["c"], chunks, io["h2d"], io["d2h"], cur)
        ev = next(e for e in t["events"] if e.cuda_event == done)
        if wait:
            cur.wait_event(ev)
        return ev


class SquadTwoPass:
    """SQuad's two-stage attention over a token sequence, through the C ABI.

    Local pass: softmax attention inside consecutive windows of ``window`` tokens (the window
    mask kind with unit = window, radius 0, no anchors: block-diagonal).  Global pass: the
    tokens at the same position of every window attend each other, with the local output as
    the value stream:

        O[a*w + p] = softmax over a' of (q_{a*w+p} . k_{a'*w+p}) O_L[a'*w + p]

    The global pass runs on the window-transposed order (position-major, row p*m + a) without
    materialising it: ``lva_window_transposed_attn`` gathers those rows through 3D tensor maps
    and stores O back in the input order.  ``window`` and ``m = n / window`` must be multiples
    of ``block_size``; inputs are [B, H, n, d] bf16 in the order whose consecutive tokens form
    the windows (e.g. after the spatiotemporal tile reorder).
    """

    def __init__(self, B, H, n, d, window, block_size=128, scale=None, device="cuda"):
        if n % window or window % block_size or (n // window) % block_size:
            raise ValueError("need n = m * window with window and m multiples of block_size")
        self.B, self.H, self.n, self.d = B, H, n, d
        self.window, self.m, self.block_size = window, n // window, block_size
        self.scale = float(scale) if scale is not None else float(torch.tensor(d ** -0.5, dtype=torch.float32))
        self.device = torch.device(device)
        kw = dict(device=self.device)
        shape = (B, H, n, d)
        self.o_local = torch.empty(shape, dtype=torch.bfloat16, **kw)
        self.o = torch.empty(shape, dtype=torch.bfloat16, **kw)
        self.lse_local = torch.empty((B, H, n), dtype=torch.float32, **kw)
        self.lse_global_t = torch.empty((B, H, n), dtype=torch.float32, **kw)   # transposed order
        nb = n // block_size
        self.csr = {}
        # local: groups of `window` consecutive tokens; global: groups of m consecutive rows of
        # the transposed order (one position across all windows)
        for name, unit in (("local", window), ("global", self.m)):
            p = lb.MaskParams(lb.LVA_MASK_WINDOW_ANCHOR, n, n, block_size, 1, unit, 0, 0, 0)
            row_ptr = torch.empty(nb + 1, dtype=torch.int32, **kw)
            col_idx = torch.empty(lb.lva_block_mask_max_nnz(p), dtype=torch.int32, **kw)
            nnz = torch.empty(1, dtype=torch.int32, **kw)
            lb.lva_build_block_mask(p, None, row_ptr, col_idx, nnz)
            # exact entry counts (read once): rows of 2-4 blocks get multi-block CTAs
            self.csr[name] = (row_ptr, col_idx[:max(1, int(nnz.item()))])

    def __call__(self, q, k, v):
        rp, ci = self.csr["local"]
        lb.lva_block_sparse_attn(q, k, v, self.o_local, self.lse_local, self.n, self.block_size, rp, ci, 1,
                                 self.scale)
        rp, ci = self.csr["global"]
        lb.lva_window_transposed_attn(q, k, self.o_local, self.o, self.lse_global_t, self.window,
                                      self.block_size, rp, ci, 1, self.scale)
        return self.o


class StaticMaskCalibrator:
    """Offline calibration of a static block mask from calibration prompts, over the C ABI.

    CalibAtt page ("Accelerating Text-to-Video Generation with Calibrated Sparse Attention"),
    section 2 A.1-A.2, for one (timestep, layer): every calibration sample (a prompt, i.e.
    one batch element of one ``add_prompt`` call) goes through

    1. ``lva_reorder_tokens`` of Q and K into tile order;
    2. ``lva_block_sparse_lse`` with the all-ones mask, for the row LSE of dense attention
       (the attention kernel's scores, maxima and sums, with no V, P V product or O);
    3. ``lva_block_energy`` -> E [B, H, nb, nb], the attention mass of every block pair;
    4. ``lva_select_blocks`` with the timestep's threshold ``eps`` -> a 0/1 mask per sample;

    and ``finish(rho)`` keeps the blocks that at least a fraction ``rho`` of the samples
    selected (``lva_aggregate_masks``).  The result, uint8 [H, nb, nb] in tile order, is the
    ``static_mask`` of ``VideoBlockSparseAttention`` with ``mask={"kind": "static"}``.
    """

    def __init__(self, B, H, d, grid, tile, block_size=128, scale=None, device="cuda"):
        self.B, self.H, self.d = B, H, d
        self.grid, self.tile, self.block_size = tuple(grid), tuple(tile), block_size
        self.n_valid = grid[0] * grid[1] * grid[2]
        self.n_pad = (self.n_valid + block_size - 1) // block_size * block_size
        self.nb = self.n_pad // block_size
        self.scale = float(scale) if scale is not None else float(torch.tensor(d ** -0.5, dtype=torch.float32))
        self.device = torch.device(device)
        kw = dict(device=self.device)
        shape = (B, H, self.n_pad, d)
        self.qk_t = torch.empty((2,) + shape, dtype=torch.bfloat16, **kw)
        self.q_t, self.k_t = self.qk_t[0], self.qk_t[1]
        self.lse = torch.empty((B, H, self.n_pad), dtype=torch.float32, **kw)
        self.energy = torch.empty((B, H, self.nb, self.nb), dtype=torch.float32, **kw)
        p = lb.MaskParams(lb.LVA_MASK_ALL, self.n_pad, self.n_valid, block_size, 1)
        self.row_ptr = torch.empty(self.nb + 1, dtype=torch.int32, **kw)
        self.col_idx = torch.empty(lb.lva_block_mask_max_nnz(p), dtype=torch.int32, **kw)
        self.nnz = torch.empty(1, dtype=torch.int32, **kw)
        lb.lva_build_block_mask(p, None, self.row_ptr, self.col_idx, self.nnz)
        self.samples = []

    def energies(self, q, k):
        """Raster-order bf16 Q, K [B, H, N, d] -> block energies E [B, H, nb, nb] (tile order)."""
        P = self.B * self.H
        for src, dst in ((q, self.q_t), (k, self.k_t)):
            lb.lva_reorder_tokens(src.reshape(P, self.n_valid, self.d), dst.view(P, self.n_pad, self.d),
                                  self.grid, self.tile, self.n_pad, inverse=False)
        lb.lva_block_sparse_lse(self.q_t, self.k_t, self.lse, self.n_valid, self.block_size, self.row_ptr,
                                self.col_idx, 1, self.scale)
        lb.lva_block_energy(self.q_t, self.k_t, self.lse, self.energy, self.n_valid, self.block_size,
                            self.row_ptr, self.col_idx, 1, self.scale)
        return self.energy

    def add_prompt(self, q, k, eps: float):
        """Select the blocks of every sample of this batch at threshold ``eps``; returns the
        per-sample masks uint8 [B, H, nb, nb]."""
        energy = self.energies(q, k)
        mask = torch.empty(energy.shape, dtype=torch.uint8, device=self.device)
        lb.lva_select_blocks(energy, mask, eps)
        self.samples.append(mask)
        return mask

    def finish(self, rho: float):
        """Aggregated static mask uint8 [H, nb, nb] over every sample added so far."""
        if not self.samples:
            raise ValueError("no calibration prompt was added")
        masks = torch.cat(self.samples, dim=0).contiguous()            # [S, H, nb, nb]
        out = torch.empty(masks.shape[1:], dtype=torch.uint8, device=self.device)
        lb.lva_aggregate_masks(masks, out, rho)
        return out
