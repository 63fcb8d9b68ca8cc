"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the library's accuracy target):
  fp32 inputs:  max |gpu - oracle| <= 1e-5
  bf16 inputs:  max |gpu - oracle| <= 2e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3
with fp32 accumulation on the GPU and fp64 in the oracle, on identical inputs
(the oracle receives the bf16 values the GPU consumed, widened to fp64).
"""
import numpy as np
import torch

FP32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_REL_L2 = 5e-3


def as64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def errors(gpu, ref):
    g, r = as64(gpu), as64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), "non-finite values in the GPU result"
    diff = g - r
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    nr = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff) / nr) if nr > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(gpu, ref, dtype, what=""):
    max_abs, rel = errors(gpu, ref)
    if dtype == torch.float32:
        assert max_abs <= FP32_ATOL, f"{what}: fp32 max abs err {max_abs:.3e} > {FP32_ATOL}"
    else:
        assert max_abs <= BF16_ATOL, f"{what}: bf16 max abs err {max_abs:.3e} > {BF16_ATOL}"
        assert rel <= BF16_REL_L2, f"{what}: bf16 rel-L2 err {rel:.3e} > {BF16_REL_L2}"
    return max_abs, rel


def assert_lse_close(gpu_lse, ref_lse, dtype, what=""):
    """lse is fp32 on the GPU: compare with an absolute bound scaled to its magnitude."""
    g, r = as64(gpu_lse), as64(ref_lse)
    tol = 1e-5 if dtype == torch.float32 else 2e-3
    err = np.abs(g - r) / np.maximum(1.0, np.abs(r))
    assert float(err.max()) <= tol, f"{what}: lse err {float(err.max()):.3e} > {tol}"
