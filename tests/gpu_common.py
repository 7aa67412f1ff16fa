"""Helpers shared by the GPU parity tests (inputs to the device, error bars)."""
from __future__ import annotations

import numpy as np

TOL_F32_ABS = 1e-4        # fp32 path: max |x - oracle|
TOL_BF16_REL_RMS = 2e-2   # bf16 path: max |x - oracle| <= 2e-2 * RMS(oracle output)


def require_cuda():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test run without a CUDA device")
    return torch


def to_dev(arr: np.ndarray, dtype: str):
    """float32 array holding exact dtype values -> CUDA tensor of that dtype (no further rounding)."""
    torch = require_cuda()
    t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def to_host(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def bound(want: np.ndarray, dtype: str) -> float:
    if dtype == "f32":
        return TOL_F32_ABS
    return TOL_BF16_REL_RMS * float(np.sqrt(np.mean(np.square(want))))


def assert_close(name: str, got: np.ndarray, want: np.ndarray, dtype: str):
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = float(np.max(np.abs(got - want)))
    b = bound(want, dtype)
    assert err <= b, f"{name}: max|err| {err:.3e} > bound {b:.3e}"
    return err, b
