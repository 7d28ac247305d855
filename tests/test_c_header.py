"""The boundary is a plain C ABI: ``include/lva.h`` compiles as strict C99 and a C program
links ``liblva.so`` and calls it (host-only paths, no GPU needed)."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "block_sparse_attention_lva_b200")
CUDA_INCLUDE = "/usr/local/cuda/include"

PROGRAM = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "lva.h"

int main(void) {
  lva_mask_params p;
  int64_t cap;
  lva_status s;
  memset(&p, 0, sizeof(p));
  p.kind = LVA_MASK_WINDOW_ANCHOR;
  p.mask_heads = 1;
  p.block_size = 128;
  p.n_pad = 32768;
  p.n_valid = 32760;
  p.window_unit_tokens = 1560;
  p.window_radius = 1;
  p.num_anchors = 4;
  p.step = 0;
  cap = lva_block_mask_max_nnz(&p);
  printf("version %d\n", lva_version());
  printf("status %s\n", lva_status_string(LVA_ERR_CAPACITY));
  printf("capacity %lld\n", (long long)cap);
  p.block_size = 96;
  printf("bad block %lld\n", (long long)lva_block_mask_max_nnz(&p));
  /* rejected on the host, before any device work */
  s = lva_reorder_tokens(NULL, NULL, 1, 0, 30, 52, 1, 8, 16, 32768, 128, 2, 0, (cudaStream_t)0);
  printf("reorder %s: %s\n", lva_status_string(s), lva_last_error_message());
  /* a non-null O is never dereferenced: validation stops at the head dim */
  s = lva_block_sparse_attn(NULL, NULL, NULL, (void*)(uintptr_t)256, NULL, 1, 12, 32768, 32760, 96, 128,
                            NULL, NULL, 0, 1, 0.125f, NULL, 1, (cudaStream_t)0);
  printf("attn %s\n", lva_status_string(s));
  s = lva_block_sparse_attn(NULL, NULL, NULL, NULL, NULL, 1, 12, 32768, 32760, 128, 128, NULL, NULL, 0, 1,
                            0.125f, NULL, 1, (cudaStream_t)0);
  printf("attn null %s: %s\n", lva_status_string(s), lva_last_error_message());
  s = lva_selftest_wait(7, (cudaStream_t)0);
  printf("selftest %s\n", lva_status_string(s));
  {
    /* the host-buffer layer step: every argument check runs before any stream or device work */
    lva_layer_shape sh;
    lva_host_step_buffers hb;
    cudaEvent_t ev[16];
    char host[64];
    memset(&sh, 0, sizeof(sh));
    memset(&hb, 0, sizeof(hb));
    memset(ev, 0, sizeof(ev));
    sh.B = 1; sh.H = 12; sh.d = 128; sh.block_size = 128; sh.T = 21; sh.Hg = 30; sh.Wg = 52;
    sh.tile_t = 1; sh.tile_h = 8; sh.tile_w = 16; sh.scale = 0.088388f;
    p.block_size = 128;
    s = lva_layer_step_host(host, host, (float*)host, NULL, &p, NULL, 1, NULL, 1, &hb, 6, 0, 0, 0, NULL);
    printf("step null %s: %s\n", lva_status_string(s), lva_last_error_message());
    sh.d = 96;
    s = lva_layer_step_host(host, host, (float*)host, &sh, &p, NULL, 1, NULL, 1, &hb, 6, 0, 0, 0, NULL);
    printf("step d96 %s\n", lva_status_string(s));
    sh.d = 128;
    s = lva_layer_step_host(host, host, (float*)host, &sh, &p, NULL, 1, NULL, 1, &hb, 6, 0, 0, 0, NULL);
    printf("step buffers %s: %s\n", lva_status_string(s), lva_last_error_message());
    hb.qkv_stage = hb.o_stage = hb.qkv_tile = (void*)(uintptr_t)256;
    hb.lse_stage = (float*)(uintptr_t)256;
    hb.row_ptr = hb.col_idx = hb.nnz = (int32_t*)(uintptr_t)256;
    hb.events = ev;
    hb.num_events = 16;
    hb.col_capacity = cap - 1;
    hb.col_len = cap - 1;
    s = lva_layer_step_host(host, host, (float*)host, &sh, &p, NULL, 1, NULL, 1, &hb, 6, 0, 0, 0, NULL);
    printf("step capacity %s\n", lva_status_string(s));
    hb.col_capacity = cap;
    hb.num_events = 2 * 6 + 1;
    s = lva_layer_step_host(host, host, (float*)host, &sh, &p, NULL, 1, NULL, 1, &hb, 6, 0, 0, 0, NULL);
    printf("step events %s: %s\n", lva_status_string(s), lva_last_error_message());
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def program():
    gcc = shutil.which("gcc")
    lib = os.path.join(PKG, "liblva.so")
    if gcc is None or not os.path.isdir(CUDA_INCLUDE):
        pytest.skip("gcc or the CUDA headers are not available")
    if not os.path.exists(lib):
        pytest.skip("liblva.so is not built")
    d = tempfile.mkdtemp()
    src, exe = os.path.join(d, "abi.c"), os.path.join(d, "abi")
    open(src, "w").write(PROGRAM)
    subprocess.check_call([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                           "-isystem", CUDA_INCLUDE, src, "-o", exe, "-L", PKG, "-llva", "-Wl,-rpath," + PKG])
    yield exe
    shutil.rmtree(d, ignore_errors=True)


def test_c_program_calls_the_library(program):
    out = subprocess.run([program], capture_output=True, text=True, timeout=120, check=True).stdout.splitlines()
    assert out[0] == "version 1"
    assert out[1] == "status LVA_ERR_CAPACITY"
    assert out[2] == f"capacity {256 * 256}"            # mask_heads * nb * nb
    assert out[3] == "bad block 0"                      # invalid parameters give no capacity
    assert out[4].startswith("reorder LVA_ERR_INVALID_ARG: reorder: grid and tile sizes must be positive")
    assert out[5] == "attn LVA_ERR_UNSUPPORTED"          # head dim 96
    assert out[6] == "attn null LVA_ERR_INVALID_ARG: attn: null pointer"
    assert out[7] == "selftest LVA_ERR_INVALID_ARG"      # unknown mode
    assert out[8] == "step null LVA_ERR_INVALID_ARG: layer_step_host: null shape, mask or buffers"
    assert out[9] == "step d96 LVA_ERR_UNSUPPORTED"
    assert out[10] == "step buffers LVA_ERR_INVALID_ARG: layer_step_host: null device buffer or event array"
    assert out[11] == "step capacity LVA_ERR_CAPACITY"       # col_capacity below the mask's maximum
    assert out[12] == ("step events LVA_ERR_INVALID_ARG: layer_step_host: too few events "
                       "(need 2 * groups + 2)")       # 6 groups of 2 heads need 14 events
