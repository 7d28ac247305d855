"""Failure detection without a GPU fault: the bounded mbarrier wait that every pipeline
kernel uses gives up and reports LVA_ERR_TIMEOUT through the device error word, and the
context stays usable afterwards (a later attention call still matches its own first run)."""
import time

import numpy as np
import pytest
import torch

from synthetic import WORKLOADS, make_qkv, mask_variants
from tests.gpu_helpers import bits, require_gpu

pytestmark = pytest.mark.gpu

LVA_ERR_TIMEOUT = 5


def _attend_tiny(lva, dev):
    w = WORKLOADS["tiny"]
    q, k, v = make_qkv(w)
    layer = lva.VideoBlockSparseAttention(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.tile, w.block_size,
                                          mask_variants(w)[0], scale=w.scale, device=dev)
    o, lse = layer(q.to(dev), k.to(dev), v.to(dev), step=0)
    return o.cpu().clone(), lse.cpu().clone()


def _timed(lva, mode):
    torch.cuda.synchronize()
    t0 = time.monotonic()
    lva.lva_selftest_wait(mode)
    status = lva.lva_device_error()
    return status, time.monotonic() - t0


def test_bounded_wait_modes_and_recovery():
    import block_sparse_attention_lva_b200 as lva
    dev = require_gpu()
    assert lva.lva_device_error() == (0, 0)
    o0, lse0 = _attend_tiny(lva, dev)
    assert lva.lva_device_error() == (0, 0)

    # the peer arrives: the wait completes and nothing is recorded
    status, secs = _timed(lva, 2)
    assert status == (0, 0) and secs < 1.0
    # the CTA's abort flag is raised: the wait gives up well before its time limit
    status, secs = _timed(lva, 1)
    assert status == (LVA_ERR_TIMEOUT, 101) and secs < 1.0
    # nothing ever arrives: the wait runs to its 2 s limit, then reports
    status, secs = _timed(lva, 0)
    assert status == (LVA_ERR_TIMEOUT, 100) and 1.9 < secs < 30.0
    # the word was cleared by the read, and the context still computes the same results
    assert lva.lva_device_error() == (0, 0)
    o1, lse1 = _attend_tiny(lva, dev)
    assert lva.lva_device_error() == (0, 0)
    assert np.array_equal(bits(o1), bits(o0)) and np.array_equal(bits(lse1), bits(lse0))
