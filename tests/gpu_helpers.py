"""Shared helpers for the GPU parity tests (comparisons, tolerances, oracle plumbing)."""
import numpy as np
import torch

# Tolerances for O and LSE against the float64 oracle, N(0,1) bf16 inputs, 1/sqrt(d) scale:
# O max|d| <= 1e-2 and mean|d| <= 1e-3 over every element (padding rows included);
# LSE max|d| <= 1e-3 over finite entries, and -inf exactly where the oracle has -inf.
O_MAX, O_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit pattern of a bf16/fp32 tensor as an integer numpy array (bit-exact compares)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    return t.numpy()


def check_o_lse(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Asserts the O / LSE tolerances; returns (max|dO|, mean|dO|, max|dLSE|)."""
    o = o_gpu.float().cpu().numpy() if isinstance(o_gpu, torch.Tensor) else o_gpu
    l = lse_gpu.float().cpu().numpy() if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    assert not np.isnan(o).any(), f"{what}: NaN in O"
    d = np.abs(o.astype(np.float64) - o_ref)
    ref_inf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l), ref_inf), f"{what}: -inf LSE pattern differs"
    fin = ~ref_inf
    dl = np.abs(l[fin].astype(np.float64) - lse_ref[fin]) if fin.any() else np.zeros(1)
    assert d.max() <= O_MAX, f"{what}: O max|d| {d.max():.3e}"
    assert d.mean() <= O_MEAN, f"{what}: O mean|d| {d.mean():.3e}"
    assert dl.max() <= LSE_MAX, f"{what}: LSE max|d| {dl.max():.3e}"
    return float(d.max()), float(d.mean()), float(dl.max())
