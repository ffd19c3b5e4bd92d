"""Helpers for comparing the CUDA path with the fp64 oracle.

Tolerances (written here once, used by every GPU parity test):
  fp32 tensors:  max |gpu - oracle| <= 1e-5
  bf16 tensors:  max |gpu - oracle| <= 1e-2 and ||gpu - oracle||_2 /
                 ||oracle||_2 <= 5e-3  (bf16 storage, fp32 accumulation)
"""
import numpy as np
import torch

F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 1e-2
BF16_REL_L2 = 5e-3


def f64(t):
    """A tensor (any device, fp32/bf16) as an exact float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()


def errors(got, want):
    got = f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(want.ravel()))
    rel = float(np.linalg.norm(diff.ravel()) / denom) if denom > 0 else float(np.linalg.norm(diff.ravel()))
    return max_abs, rel


def assert_close(got, want, dtype, what=""):
    max_abs, rel = errors(got, want)
    if dtype == torch.float32:
        assert max_abs <= F32_MAX_ABS, f"{what}: max abs {max_abs:.3e} > {F32_MAX_ABS}"
    else:
        assert max_abs <= BF16_MAX_ABS, f"{what}: max abs {max_abs:.3e} > {BF16_MAX_ABS}"
        assert rel <= BF16_REL_L2, f"{what}: rel L2 {rel:.3e} > {BF16_REL_L2}"
    assert np.isfinite(f64(got) if isinstance(got, torch.Tensor) else got).all(), what
    return max_abs, rel
