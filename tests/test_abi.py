"""The C-ABI library loads and exports every declared symbol; host-side argument checks
reject bad calls before anything reaches a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lva.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lva_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import block_sparse_attention_lva_b200 as lva
    lib = ctypes.CDLL(lva.LIB_PATH)
    names = _declared()
    assert "lva_block_sparse_attn" in names and "lva_build_block_mask" in names and "lva_reorder_tokens" in names
    for n in names:
        assert hasattr(lib, n), n
    from block_sparse_attention_lva_b200._binding import SIGNATURES
    assert set(SIGNATURES) == set(names)


def test_status_strings_and_version():
    from block_sparse_attention_lva_b200._binding import lib
    assert lib.lva_version() == 1
    assert lib.lva_status_string(0) == b"LVA_OK"
    assert lib.lva_status_string(3) == b"LVA_ERR_CAPACITY"


def test_mask_param_checks():
    import block_sparse_attention_lva_b200 as lva
    P = lva.MaskParams
    assert lva.lva_block_mask_max_nnz(P(lva.LVA_MASK_WINDOW_ANCHOR, 32768, 32760, 128, 1, 1560, 1, 4, 0)) == 256 * 256
    assert lva.lva_block_mask_max_nnz(P(lva.LVA_MASK_STATIC, 256, 256, 64, 12)) == 12 * 16
    bad = [P(0, 1000, 1000, 128),              # n_pad not a multiple of the block
           P(0, 1024, 0, 128),                 # no real tokens
           P(0, 1024, 2000, 128),              # n_valid > n_pad
           P(0, 1024, 1024, 96),               # unsupported block size
           P(0, 1024, 1024, 128, 2, 1, 1),     # parametric kind with 2 mask heads
           P(0, 1024, 1024, 128, 1, 0, 1),     # window unit 0
           P(0, 1024, 1024, 128, 1, 128, -1),  # negative radius
           P(3, 1024, 1024, 128, 1, group_blocks=0),
           P(9, 1024, 1024, 128)]
    for p in bad:
        assert lva.lva_block_mask_max_nnz(p) == 0, p


def test_attn_argument_checks_fail_before_launch():
    from block_sparse_attention_lva_b200._binding import lib
    vp = ctypes.c_void_p(16)
    call = lambda **kw: lib.lva_block_sparse_attn(
        kw.get("q", vp), vp, vp, vp, vp, kw.get("B", 1), kw.get("H", 2), kw.get("n_pad", 256),
        kw.get("n_valid", 256), kw.get("d", 128), kw.get("bs", 128), vp, vp, 10, kw.get("mh", 1),
        ctypes.c_float(0.1), kw.get("qs", None), kw.get("sh", 1), None)
    assert call(d=96) == 2                       # unsupported head dim
    assert call(bs=32) == 2                      # unsupported block size
    assert call(n_pad=200) == 1                  # not a multiple of the block
    assert call(n_valid=300) == 1
    assert call(mh=3) == 1                       # mask heads must be 1 or H
    assert call(q=ctypes.c_void_p(18)) == 1      # misaligned pointer
    assert b"aligned" in lib.lva_last_error_message()
    assert call(q=None) == 1
    assert call(qs=vp, sh=3) == 1                # src_heads must be 1 or H
    f = lib.lva_broadcast_blocks
    assert f(vp, vp, 1, 2, 256, 96, 128, vp, 1, None) == 2     # head dim
    assert f(vp, vp, 1, 2, 256, 128, 128, None, 1, None) == 1  # null map
    assert f(vp, vp, 1, 2, 200, 128, 128, vp, 1, None) == 1    # n_pad


def test_reorder_argument_checks_fail_before_launch():
    from block_sparse_attention_lva_b200._binding import lib
    vp = ctypes.c_void_p(64)
    f = lib.lva_reorder_tokens
    assert f(vp, vp, 2, 4, 8, 8, 1, 4, 4, 200, 64, 2, 0, None) == 1     # n_pad < T*H*W
    assert f(vp, vp, 2, 4, 8, 8, 1, 4, 4, 256, 64, 3, 0, None) == 1     # elem_bytes
    assert f(vp, vp, 2, 4, 8, 8, 0, 4, 4, 256, 64, 2, 0, None) == 1     # zero tile
    assert f(None, vp, 2, 4, 8, 8, 1, 4, 4, 256, 64, 2, 0, None) == 1   # null
    assert f(vp, vp, 0, 4, 8, 8, 1, 4, 4, 256, 64, 2, 0, None) == 0     # no planes: no-op
    # grid limit: one thread per (row, element chunk), 256-thread blocks, gridDim.x < 2^31
    # (planes = 0 returns after the size checks, before any pointer is used)
    assert f(vp, vp, 0, 1, 1, 1, 1, 1, 1, 1 << 30, 511, 2, 0, None) == 0
    assert f(vp, vp, 0, 1, 1, 1, 1, 1, 1, 1 << 30, 512, 2, 0, None) == 2
    assert b"too large" in lib.lva_last_error_message()
    assert f(vp, vp, 0, 1, 1, 1, 1, 1, 1, 1 << 30, 512, 4, 0, None) == 2


def test_mask_capacity_check():
    from block_sparse_attention_lva_b200._binding import LvaMaskParams, lib
    p = LvaMaskParams(2, 1, 128, 1024, 1024, 1, 0, 0, 0, 1)
    vp = ctypes.c_void_p(64)
    assert lib.lva_build_block_mask(ctypes.byref(p), None, vp, vp, 63, vp, None) == 3
    assert b"col_capacity" in lib.lva_last_error_message()


def test_calibration_argument_checks_fail_before_launch():
    from block_sparse_attention_lva_b200._binding import lib
    vp = ctypes.c_void_p(64)
    energy = lambda **kw: lib.lva_block_energy(
        kw.get("q", vp), vp, vp, vp, 1, 2, kw.get("n_pad", 256), kw.get("n_valid", 256), kw.get("d", 128),
        kw.get("bs", 128), vp, vp, 4, kw.get("mh", 1), ctypes.c_float(0.1), None)
    assert energy(d=96) == 2
    assert energy(bs=32) == 2
    assert energy(n_pad=200) == 1
    assert energy(mh=3) == 1
    assert energy(q=ctypes.c_void_p(72)) == 1      # not 16-byte aligned
    assert energy(q=None) == 1
    sel = lambda rows, nb, eps: lib.lva_select_blocks(vp, vp, rows, nb, ctypes.c_double(eps), None)
    assert sel(4, 0, 0.5) == 1                     # no key blocks
    assert sel(4, 5000, 0.5) == 2                  # beyond the supported row length
    assert sel(4, 16, 1.5) == 1 and sel(4, 16, -0.1) == 1
    assert sel(0, 16, 0.5) == 0                    # no rows: no-op
    assert lib.lva_select_blocks(None, vp, 4, 16, ctypes.c_double(0.5), None) == 1
    agg = lambda prompts, count, rho: lib.lva_aggregate_masks(vp, vp, prompts, count, ctypes.c_double(rho), None)
    assert agg(0, 16, 0.5) == 1
    assert agg(2, 16, 1.5) == 1
    assert agg(2, 0, 0.5) == 0


def test_window_transposed_attn_argument_checks():
    from block_sparse_attention_lva_b200._binding import lib
    vp = ctypes.c_void_p(64)
    call = lambda n, w, bs=128, d=128: lib.lva_window_transposed_attn(
        vp, vp, vp, vp, vp, 1, 2, n, d, w, bs, vp, vp, 4, 1, ctypes.c_float(0.1), None)
    assert call(32768, 300) == 1            # n not a multiple of the window
    assert call(32768, 512) == 1            # m = 64 windows: not a multiple of the block
    assert call(32768, 256, bs=32) == 2     # unsupported block size
    assert call(32768, 256, d=96) == 2      # unsupported head dim
    assert lib.lva_window_transposed_attn(vp, vp, vp, None, vp, 1, 2, 32768, 128, 256, 128, vp, vp, 4, 1,
                                          ctypes.c_float(0.1), None) == 1


def test_selftest_wait_rejects_unknown_mode():
    from block_sparse_attention_lva_b200._binding import lib
    assert lib.lva_selftest_wait(3, None) == 1
    assert lib.lva_selftest_wait(-1, None) == 1
