"""ctypes binding of ``liblva.so`` (the C ABI of ``include/lva.h``).

Argument marshalling only: each function takes torch tensors that live on the current
CUDA device, passes their device pointers and the current stream to the C function of the
same name, and raises ``LvaError`` on a non-OK status.  All computation happens in the
library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblva.so")

LVA_OK = 0
LVA_MASK_WINDOW_ANCHOR = 0
LVA_MASK_STATIC = 1
LVA_MASK_ALL = 2
LVA_MASK_TWO_STAGE = 3
LVA_MASK_LVSA_FRAMES = 4

STATUS_NAMES = {0: "LVA_OK", 1: "LVA_ERR_INVALID_ARG", 2: "LVA_ERR_UNSUPPORTED",
                3: "LVA_ERR_CAPACITY", 4: "LVA_ERR_CUDA", 5: "LVA_ERR_TIMEOUT"}

# Every symbol the header declares, with its ctypes signature.
_c_i64, _c_int, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p


class LvaMaskParams(ctypes.Structure):
    """Mirror of ``lva_mask_params``."""
    _fields_ = [("kind", ctypes.c_int), ("mask_heads", ctypes.c_int), ("block_size", ctypes.c_int),
                ("n_pad", ctypes.c_int64), ("n_valid", ctypes.c_int64),
                ("window_unit_tokens", ctypes.c_int64), ("window_radius", ctypes.c_int),
                ("num_anchors", ctypes.c_int), ("step", ctypes.c_int), ("group_blocks", ctypes.c_int),
                ("budget_frames", ctypes.c_int)]


class LvaLayerShape(ctypes.Structure):
    """Mirror of ``lva_layer_shape``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("block_size", ctypes.c_int),
                ("T", ctypes.c_int), ("Hg", ctypes.c_int), ("Wg", ctypes.c_int), ("tile_t", ctypes.c_int),
                ("tile_h", ctypes.c_int), ("tile_w", ctypes.c_int), ("scale", ctypes.c_float)]


class LvaHostStepBuffers(ctypes.Structure):
    """Mirror of ``lva_host_step_buffers``."""
    _fields_ = [("qkv_stage", ctypes.c_void_p), ("o_stage", ctypes.c_void_p), ("lse_stage", ctypes.c_void_p),
                ("qkv_tile", ctypes.c_void_p), ("o_tile", ctypes.c_void_p), ("row_ptr", ctypes.c_void_p),
                ("col_idx", ctypes.c_void_p), ("col_capacity", ctypes.c_int64), ("col_len", ctypes.c_int64),
                ("nnz", ctypes.c_void_p), ("events", ctypes.POINTER(ctypes.c_void_p)), ("num_events", ctypes.c_int)]


SIGNATURES = {
    "lva_status_string": (ctypes.c_char_p, [_c_int]),
    "lva_last_error_message": (ctypes.c_char_p, []),
    "lva_version": (_c_int, []),
    "lva_reorder_tokens": (_c_int, [_vp, _vp, _c_i64, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                    _c_i64, _c_i64, _c_int, _c_int, _vp]),
    "lva_block_mask_max_nnz": (_c_i64, [ctypes.POINTER(LvaMaskParams)]),
    "lva_build_block_mask": (_c_int, [ctypes.POINTER(LvaMaskParams), _vp, _vp, _vp, _c_i64, _vp, _vp]),
    "lva_block_mask_workspace_bytes": (_c_i64, [ctypes.POINTER(LvaMaskParams)]),
    "lva_build_block_mask_ws": (_c_int, [ctypes.POINTER(LvaMaskParams), _vp, _vp, _vp, _c_i64, _vp, _vp, _c_i64,
                                         _vp]),
    "lva_build_block_mask_noalloc": (_c_int, [ctypes.POINTER(LvaMaskParams), _vp, _vp, _vp, _c_i64, _vp, _vp]),
    "lva_block_sparse_attn": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_i64, _c_int,
                                       _c_int, _vp, _vp, _c_i64, _c_int, ctypes.c_float, _vp, _c_int, _vp]),
    "lva_block_sparse_lse": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_i64, _c_int, _c_int, _vp, _vp,
                                      _c_i64, _c_int, ctypes.c_float, _vp]),
    "lva_block_sparse_attn_raster": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_i64, _c_int,
                                              _c_int, _vp, _vp, _c_i64, _c_int, ctypes.c_float, _c_int, _c_int,
                                              _c_int, _c_int, _c_int, _c_int, _vp]),
    "lva_window_transposed_attn": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                            _c_int, _vp, _vp, _c_i64, _c_int, ctypes.c_float, _vp]),
    "lva_broadcast_blocks": (_c_int, [_vp, _vp, _c_int, _c_int, _c_i64, _c_int, _c_int, _vp, _c_int, _vp]),
    "lva_block_energy": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_i64, _c_i64, _c_int, _c_int,
                                  _vp, _vp, _c_i64, _c_int, ctypes.c_float, _vp]),
    "lva_select_blocks": (_c_int, [_vp, _vp, _c_i64, _c_int, ctypes.c_double, _vp]),
    "lva_aggregate_masks": (_c_int, [_vp, _vp, _c_int, _c_i64, ctypes.c_double, _vp]),
    "lva_layer_step_host": (_c_int, [_vp, _vp, _vp, ctypes.POINTER(LvaLayerShape), ctypes.POINTER(LvaMaskParams),
                                     _vp, _c_int, _vp, _c_int, ctypes.POINTER(LvaHostStepBuffers), _c_int, _vp, _vp,
                                     _vp, ctypes.POINTER(ctypes.c_void_p)]),
    "lva_device_error": (_c_int, [_vp, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "lva_selftest_wait": (_c_int, [_c_int, _vp]),
}


class LvaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA library first "
            "(python -c 'import __graft_entry__ as g; g.build()' or python block_sparse_attention_lva_b200/build.py)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int):
    if status != LVA_OK:
        raise LvaError(status, lib.lva_last_error_message().decode())


def _stream(device=None) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _cuda_tensor(t, name: str, dtype=None, numel: int = None):
    """Checks that ``t`` is a contiguous CUDA tensor on the current device (of ``dtype``, with
    >= ``numel`` elements).  The library launches on the current device, so a tensor of
    another device would hand its kernels a foreign address."""
    import torch
    _need(t is not None and t.is_cuda, f"{name} must be a CUDA tensor")
    current = torch.cuda.current_device()
    _need(t.device.index == current, f"{name} is on cuda:{t.device.index}, the current device is cuda:{current}")
    _need(t.is_contiguous(), f"{name} must be contiguous")
    if dtype is not None:
        _need(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None:
        _need(t.numel() >= numel, f"{name} has {t.numel()} elements, needs {numel}")


@dataclass
class MaskParams:
    """Python view of ``lva_mask_params``."""
    kind: int
    n_pad: int
    n_valid: int
    block_size: int = 128
    mask_heads: int = 1
    window_unit_tokens: int = 1
    window_radius: int = 0
    num_anchors: int = 0
    step: int = 0
    group_blocks: int = 1
    budget_frames: int = 1

    def to_c(self) -> LvaMaskParams:
        return LvaMaskParams(self.kind, self.mask_heads, self.block_size, self.n_pad, self.n_valid,
                             self.window_unit_tokens, self.window_radius, self.num_anchors, self.step,
                             self.group_blocks, self.budget_frames)


def lva_version() -> int:
    return lib.lva_version()


def lva_reorder_tokens(src, dst, grid, tile, n_pad: int, inverse: bool = False):
    """Tile-order gather (``inverse=False``: src [P, N, row] -> dst [P, n_pad, row]) or the
    inverse scatter (src [P, n_pad, row] -> dst [P, N, row]); rows are the trailing dims."""
    T, H, W = grid
    n = T * H * W
    planes = src.shape[0]
    row_elems = 1
    for x in src.shape[2:]:
        row_elems *= x
    _cuda_tensor(src, "src", numel=planes * (n_pad if inverse else n) * row_elems)
    _cuda_tensor(dst, "dst", dtype=src.dtype, numel=planes * (n if inverse else n_pad) * row_elems)
    _need(src.shape[1] == (n_pad if inverse else n), "src rows must be n_pad (inverse) or T*H*W")
    _check(lib.lva_reorder_tokens(_ptr(src), _ptr(dst), planes, T, H, W, tile[0], tile[1], tile[2],
                                  n_pad, row_elems, src.element_size(), int(bool(inverse)),
                                  ctypes.c_void_p(_stream(src.device))))
    return dst


def lva_block_mask_max_nnz(params: MaskParams) -> int:
    cp = params.to_c()
    return lib.lva_block_mask_max_nnz(ctypes.byref(cp))


def lva_build_block_mask(params: MaskParams, dense_mask, row_ptr, col_idx, nnz_out):
    """Build the CSR of a block mask on the GPU into caller-owned int32 buffers."""
    import torch
    nb = params.n_pad // params.block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, params.mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    _cuda_tensor(nnz_out, "nnz_out", torch.int32, 1)
    if params.kind == LVA_MASK_STATIC:
        _cuda_tensor(dense_mask, "dense_mask", torch.uint8, params.mask_heads * nb * nb)
    else:
        dense_mask = None
    cp = params.to_c()
    _check(lib.lva_build_block_mask(ctypes.byref(cp), _ptr(dense_mask), _ptr(row_ptr), _ptr(col_idx),
                                    col_idx.numel(), _ptr(nnz_out),
                                    ctypes.c_void_p(_stream(row_ptr.device))))
    return row_ptr, col_idx, nnz_out


def lva_block_mask_workspace_bytes(params: MaskParams) -> int:
    cp = params.to_c()
    return lib.lva_block_mask_workspace_bytes(ctypes.byref(cp))


def lva_build_block_mask_ws(params: MaskParams, dense_mask, row_ptr, col_idx, nnz_out, workspace):
    """``lva_build_block_mask`` with a caller-owned device workspace (uint8 tensor of at least
    ``lva_block_mask_workspace_bytes(params)`` bytes; may be None when that is 0)."""
    import torch
    nb = params.n_pad // params.block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, params.mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    _cuda_tensor(nnz_out, "nnz_out", torch.int32, 1)
    if params.kind == LVA_MASK_STATIC:
        _cuda_tensor(dense_mask, "dense_mask", torch.uint8, params.mask_heads * nb * nb)
    else:
        dense_mask = None
    ws_bytes = 0
    if workspace is not None:
        _cuda_tensor(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    cp = params.to_c()
    _check(lib.lva_build_block_mask_ws(ctypes.byref(cp), _ptr(dense_mask), _ptr(row_ptr), _ptr(col_idx),
                                       col_idx.numel(), _ptr(nnz_out), _ptr(workspace), ws_bytes,
                                       ctypes.c_void_p(_stream(row_ptr.device))))
    return row_ptr, col_idx, nnz_out


def lva_build_block_mask_noalloc(params: MaskParams, dense_mask, row_ptr, col_idx, nnz_out):
    """``lva_build_block_mask_ws`` with the scratch in the library's own 16 MiB device array
    (no workspace argument; nothing is allocated by the call)."""
    import torch
    nb = params.n_pad // params.block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, params.mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    _cuda_tensor(nnz_out, "nnz_out", torch.int32, 1)
    if params.kind == LVA_MASK_STATIC:
        _cuda_tensor(dense_mask, "dense_mask", torch.uint8, params.mask_heads * nb * nb)
    else:
        dense_mask = None
    cp = params.to_c()
    _check(lib.lva_build_block_mask_noalloc(ctypes.byref(cp), _ptr(dense_mask), _ptr(row_ptr), _ptr(col_idx),
                                            col_idx.numel(), _ptr(nnz_out), ctypes.c_void_p(_stream(row_ptr.device))))
    return row_ptr, col_idx, nnz_out


def _check_query_src(query_src, H, nb):
    import torch
    _cuda_tensor(query_src, "query_src", torch.int32)
    _need(query_src.dim() == 2 and query_src.shape[0] in (1, H) and query_src.shape[1] == nb,
          f"query_src must have shape [1 or {H}, {nb}]")


def lva_block_sparse_attn(q, k, v, o, lse, n_valid: int, block_size: int, row_ptr, col_idx,
                          mask_heads: int, scale: float, query_src=None):
    """O, LSE of block-sparse softmax attention over the CSR-listed key blocks.  With
    ``query_src`` ([1 or H, nb] int32), blocks whose source is another block are skipped."""
    import torch
    B, H, n_pad, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _cuda_tensor(t, name, torch.bfloat16)
        _need(tuple(t.shape) == (B, H, n_pad, d), f"{name} must have shape {(B, H, n_pad, d)}")
    _cuda_tensor(lse, "lse", torch.float32, B * H * n_pad)
    nb = n_pad // block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    src_heads = 1
    if query_src is not None:
        _check_query_src(query_src, H, nb)
        src_heads = query_src.shape[0]
    _check(lib.lva_block_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_pad, n_valid,
                                     d, block_size, _ptr(row_ptr), _ptr(col_idx), col_idx.numel(),
                                     mask_heads, ctypes.c_float(scale), _ptr(query_src), src_heads,
                                     ctypes.c_void_p(_stream(q.device))))
    return o, lse


def lva_block_sparse_lse(q, k, lse, n_valid: int, block_size: int, row_ptr, col_idx, mask_heads: int,
                         scale: float):
    """Row log-sum-exp [B, H, n_pad] (fp32) of block-sparse attention, without O (V unused)."""
    import torch
    B, H, n_pad, d = q.shape
    for name, t in (("q", q), ("k", k)):
        _cuda_tensor(t, name, torch.bfloat16)
        _need(tuple(t.shape) == (B, H, n_pad, d), f"{name} must have shape {(B, H, n_pad, d)}")
    _cuda_tensor(lse, "lse", torch.float32, B * H * n_pad)
    nb = n_pad // block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    _check(lib.lva_block_sparse_lse(_ptr(q), _ptr(k), _ptr(lse), B, H, n_pad, n_valid, d, block_size,
                                    _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), mask_heads,
                                    ctypes.c_float(scale), ctypes.c_void_p(_stream(q.device))))
    return lse


def lva_block_sparse_attn_raster(q, k, v, o_raster, lse, n_valid: int, block_size: int, row_ptr, col_idx,
                                 mask_heads: int, scale: float, grid, tile):
    """Block-sparse attention on tile-order Q, K, V with O written in raster order
    ([B, H, n_valid, d]); LSE stays in tile order ([B, H, n_pad])."""
    import torch
    B, H, n_pad, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _cuda_tensor(t, name, torch.bfloat16)
        _need(tuple(t.shape) == (B, H, n_pad, d), f"{name} must have shape {(B, H, n_pad, d)}")
    _cuda_tensor(o_raster, "o_raster", torch.bfloat16, B * H * n_valid * d)
    _cuda_tensor(lse, "lse", torch.float32, B * H * n_pad)
    nb = n_pad // block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    T, Hg, Wg = grid
    tt, th, tw = tile
    _check(lib.lva_block_sparse_attn_raster(_ptr(q), _ptr(k), _ptr(v), _ptr(o_raster), _ptr(lse), B, H, n_pad,
                                            n_valid, d, block_size, _ptr(row_ptr), _ptr(col_idx),
                                            col_idx.numel(), mask_heads, ctypes.c_float(scale), T, Hg, Wg,
                                            tt, th, tw, ctypes.c_void_p(_stream(q.device))))
    return o_raster, lse


def lva_window_transposed_attn(q, k, v, o, lse, window: int, block_size: int, row_ptr, col_idx,
                               mask_heads: int, scale: float):
    """Block-sparse attention on the window-transposed order of q, k, v ([B, H, n, d], read in
    place); O is stored in the input order, LSE ([B, H, n]) in the transposed order."""
    import torch
    B, H, n, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _cuda_tensor(t, name, torch.bfloat16)
        _need(tuple(t.shape) == (B, H, n, d), f"{name} must have shape {(B, H, n, d)}")
    _cuda_tensor(lse, "lse", torch.float32, B * H * n)
    nb = n // block_size
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    _check(lib.lva_window_transposed_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n, d, window,
                                          block_size, _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), mask_heads,
                                          ctypes.c_float(scale), ctypes.c_void_p(_stream(q.device))))
    return o, lse


def lva_broadcast_blocks(o, lse, block_size: int, query_src):
    """Copy O rows and LSE of anchor blocks into the blocks that name them in ``query_src``."""
    import torch
    B, H, n_pad, d = o.shape
    _cuda_tensor(o, "o", torch.bfloat16)
    _cuda_tensor(lse, "lse", torch.float32, B * H * n_pad)
    _check_query_src(query_src, H, n_pad // block_size)
    _check(lib.lva_broadcast_blocks(_ptr(o), _ptr(lse), B, H, n_pad, d, block_size, _ptr(query_src),
                                    query_src.shape[0], ctypes.c_void_p(_stream(o.device))))
    return o, lse


def lva_block_energy(q, k, lse, energy, n_valid: int, block_size: int, row_ptr, col_idx,
                     mask_heads: int, scale: float):
    """Block energies [B, H, nb, nb] (fp32) of softmax attention, given the dense-pass LSE."""
    import torch
    B, H, n_pad, d = q.shape
    for name, t in (("q", q), ("k", k)):
        _cuda_tensor(t, name, torch.bfloat16)
        _need(tuple(t.shape) == (B, H, n_pad, d), f"{name} must have shape {(B, H, n_pad, d)}")
    nb = n_pad // block_size
    _cuda_tensor(lse, "lse", torch.float32, B * H * n_pad)
    _cuda_tensor(energy, "energy", torch.float32, B * H * nb * nb)
    _cuda_tensor(row_ptr, "row_ptr", torch.int32, mask_heads * nb + 1)
    _cuda_tensor(col_idx, "col_idx", torch.int32)
    _check(lib.lva_block_energy(_ptr(q), _ptr(k), _ptr(lse), _ptr(energy), B, H, n_pad, n_valid, d,
                                block_size, _ptr(row_ptr), _ptr(col_idx), col_idx.numel(), mask_heads,
                                ctypes.c_float(scale), ctypes.c_void_p(_stream(q.device))))
    return energy


def lva_select_blocks(energy, mask, eps: float):
    """0/1 mask (uint8, same shape) of the fewest key blocks reaching ``eps`` of each row's
    energy; the last axis is the key block axis."""
    import torch
    _cuda_tensor(energy, "energy", torch.float32)
    _cuda_tensor(mask, "mask", torch.uint8, energy.numel())
    nb = energy.shape[-1]
    _check(lib.lva_select_blocks(_ptr(energy), _ptr(mask), energy.numel() // nb, nb, ctypes.c_double(eps),
                                 ctypes.c_void_p(_stream(energy.device))))
    return mask


def lva_aggregate_masks(masks, out, rho: float):
    """Blocks kept by at least a fraction ``rho`` of the prompt masks ``masks[P, ...]``."""
    import torch
    _cuda_tensor(masks, "masks", torch.uint8)
    _cuda_tensor(out, "out", torch.uint8)
    _need(masks.dim() >= 1 and masks.shape[0] >= 1 and out.numel() == masks[0].numel(),
          "out must have as many elements as one prompt's mask masks[p]")
    _check(lib.lva_aggregate_masks(_ptr(masks), _ptr(out), masks.shape[0], out.numel(), ctypes.c_double(rho),
                                   ctypes.c_void_p(_stream(masks.device))))
    return out


def lva_layer_step_host(qkv_host, o_host, lse_host, shape: LvaLayerShape, params: "MaskParams", dense_mask,
                        build_mask: bool, query_src, bufs: LvaHostStepBuffers, head_groups: int, h2d, d2h,
                        compute=None) -> int:
    """Enqueue one layer step from pinned host buffers (``lva_layer_step_host``); returns the
    raw handle of the event that completes when ``o_host`` and ``lse_host`` hold the results.
    ``h2d`` / ``d2h`` / ``compute`` are torch streams (compute: the current stream)."""
    import torch
    B, H, d = shape.B, shape.H, shape.d
    N = shape.T * shape.Hg * shape.Wg
    for name, t, shp, dt in (("qkv_host", qkv_host, (3, B, H, N, d), torch.bfloat16),
                             ("o_host", o_host, (B, H, N, d), torch.bfloat16),
                             ("lse_host", lse_host, (B, H, params.n_pad), torch.float32)):
        _need(tuple(t.shape) == shp and t.dtype == dt and t.is_contiguous() and not t.is_cuda,
              f"{name} must be a contiguous host {dt} tensor of shape {shp}")
    if params.kind == LVA_MASK_STATIC and build_mask:
        nb = params.n_pad // params.block_size
        _cuda_tensor(dense_mask, "dense_mask", torch.uint8, params.mask_heads * nb * nb)
    src_heads = 1
    if query_src is not None:
        _check_query_src(query_src, H, params.n_pad // params.block_size)
        src_heads = query_src.shape[0]
    compute = torch.cuda.current_stream() if compute is None else compute
    cp = params.to_c()
    done = ctypes.c_void_p(0)
    _check(lib.lva_layer_step_host(_ptr(qkv_host), _ptr(o_host), _ptr(lse_host), ctypes.byref(shape),
                                   ctypes.byref(cp), _ptr(dense_mask) if params.kind == LVA_MASK_STATIC else None,
                                   int(bool(build_mask)), _ptr(query_src), src_heads, ctypes.byref(bufs),
                                   int(head_groups), ctypes.c_void_p(compute.cuda_stream),
                                   ctypes.c_void_p(h2d.cuda_stream), ctypes.c_void_p(d2h.cuda_stream),
                                   ctypes.byref(done)))
    return done.value


def lva_device_error(stream=None):
    """(status, detail) of the kernel error word of the current device; clears it."""
    st, det = ctypes.c_int(0), ctypes.c_int(0)
    s = _stream() if stream is None else stream
    _check(lib.lva_device_error(ctypes.c_void_p(s), ctypes.byref(st), ctypes.byref(det)))
    return st.value, det.value


def lva_selftest_wait(mode: int, stream=None):
    """Runs the bounded-wait self-test kernel (mode 0: runs out, 1: aborted, 2: completes) on
    the current stream; read the outcome with ``lva_device_error``."""
    s = _stream() if stream is None else stream
    _check(lib.lva_selftest_wait(int(mode), ctypes.c_void_p(s)))
