"""The attention kernel's FMA-pipe exp2 (ptx.cuh, exp2_poly_f2), replayed step by step in
float32 on the CPU: its error bound against exp2 in float64, the clamp region, and that the
Remez fit script reproduces the kernel's coefficients (no GPU)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_lva_b200", "csrc")


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = src[src.index("exp2_poly_f2(uint64_t x)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([-+0-9.e]+)f, \1f\)", body)]
    vals = [v for v in vals if abs(v) < 2.0]            # drop the 1.5 * 2^23 rounding constant
    c3, c2, c1, c0 = vals
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _emulate(x):
    """The kernel's steps in float32 (FMA evaluated in float64 then rounded once)."""
    c0, c1, c2, c3 = _kernel_coefficients()
    f32 = np.float32
    xc = np.maximum(x.astype(f32), f32(-125.0))
    magic = f32(12582912.0)
    t = (xc + magic).astype(f32)
    f = (xc - (t - magic).astype(f32)).astype(f32)
    fma = lambda a, b, c: (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(f32)
    q = fma(np.full_like(f, c3), f, c2)
    q = fma(q, f, c1)
    q = fma(q, f, c0)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) \
        & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(f32)


def test_error_bound_on_working_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    x = np.concatenate([x, np.float32([-0.5, 0.5, -1.5, 1e-8, -1e-8, 0.0, 7.999999])])
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()           # fit: 7.5e-5, plus float32 rounding


def test_clamp_region_is_negligible():
    x = np.float32([-126.0, -200.0, -1e30, -3.4e38])
    got = _emulate(x)
    assert np.all(got > 0) and np.all(got < 3e-38)


def test_fit_script_reproduces_kernel_constants():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    coef, err = fit.remez()
    assert err < 8e-5
    got = np.array(_kernel_coefficients(), dtype=np.float64)
    assert np.allclose(got, coef.astype(np.float32).astype(np.float64), rtol=0, atol=1e-9)
