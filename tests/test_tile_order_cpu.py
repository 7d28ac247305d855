"""The closed-form tile-order -> raster map shared by the reorder kernels and the attention
epilogue (csrc/tile_order.cuh, host-compilable), compiled for the CPU with g++ and compared
entry by entry with the oracle's permutation built by explicit loops over tiles."""
import ctypes
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle.reorder import tile_permutation

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "block_sparse_attention_lva_b200", "csrc")

WRAPPER = r"""
#define __host__
#define __device__
#define __forceinline__ inline
#include "tile_order.cuh"
extern "C" void perm(unsigned T, unsigned H, unsigned W, unsigned tt, unsigned th, unsigned tw,
                     unsigned n, unsigned* out) {
  const lva::Grid3 g{T, H, W, tt, th, tw};
  for (unsigned k = 0; k < n; ++k) out[k] = lva::tile_order_to_raster(k, g);
}
"""


@pytest.fixture(scope="module")
def closed_form():
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ is not available")
    d = tempfile.mkdtemp()
    src, lib = os.path.join(d, "perm.cpp"), os.path.join(d, "libperm.so")
    open(src, "w").write(WRAPPER)
    subprocess.check_call([gxx, "-O1", "-std=c++17", "-shared", "-fPIC", "-I", HEADER_DIR, src, "-o", lib])
    so = ctypes.CDLL(lib)
    so.perm.argtypes = [ctypes.c_uint] * 7 + [ctypes.c_void_p]

    def run(T, H, W, tt, th, tw):
        n = T * H * W
        out = np.empty(n, dtype=np.uint32)
        so.perm(T, H, W, tt, th, tw, n, out.ctypes.data)
        return out
    yield run
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("grid,tile", [
    ((4, 8, 8), (1, 4, 4)),          # tiny workload
    ((21, 30, 52), (1, 8, 16)),      # small: partial tile rows and columns
    ((21, 45, 80), (1, 8, 16)),      # large
    ((3, 10, 21), (1, 4, 8)),        # partial tiles everywhere
    ((5, 9, 13), (2, 3, 5)),         # depth-2 tiles, last slab partial
    ((7, 1, 1), (3, 1, 1)),          # one token per frame
    ((1, 256, 512), (1, 256, 1)),    # SQuad window transpose: m = 256 windows of 512
    ((2, 6, 6), (4, 8, 8)),          # a tile larger than the grid
])
def test_closed_form_matches_loop_permutation(closed_form, grid, tile):
    got = closed_form(*grid, *tile)
    ref = tile_permutation(*grid, *tile)
    assert np.array_equal(got, ref.astype(np.uint32))


def test_window_transpose_closed_form():
    # grid (1, m, w) with tiles (1, m, 1): transposed row k = p*m + a is token a*w + p
    m, w = 8, 6
    ref = tile_permutation(1, m, w, 1, m, 1)
    k = np.arange(m * w)
    assert np.array_equal(ref, (k % m) * w + k // m)
