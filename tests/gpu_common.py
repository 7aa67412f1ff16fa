"""Helpers shared by the GPU parity tests: inputs to the device and error bars.

Two bars are used (the reasoning is in the design notes, "Parity bars"):

* stated: fp32 path max|x - oracle| <= 1e-4; bf16 inputs max|x - oracle| <=
  2e-2 * RMS(oracle output).
* bf16 storage: the tensor-core path stores Q_dyn, Z and Y as bf16, as three
  chained bf16 SDPA calls would.  Every output is a convex combination of
  rows R (V for Q_dyn and Z, the oracle's Z for Y), so per head
      max|x - oracle| <= 2e-2 * RMS(oracle) + c * 2^-9 * max|R_h|,
  with c = 2 for the encodes (two rounding steps of 2^-9 at the scale of the
  averaged rows) and c = 16 for the decode output (the rounding of Q_dyn
  moves the decode logits by up to 2^-9 |k| |q| and is amplified by sharp
  decode softmaxes on large-norm tokens).  Where the stated bar can hold at
  all for bf16 storage, it is asserted as well.
"""
from __future__ import annotations

import numpy as np

TOL_F32_ABS = 1e-4
TOL_BF16_REL_RMS = 2e-2


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


def encode_kernels(B: int, H: int, N: int, tensor_cores: bool = True) -> list:
    """The kernels of one encode: the tensor-core encode is followed by a
    log-sum-exp merge unless it runs one CTA per head (then it writes its
    result itself); the CUDA-core encode always merges."""
    if not tensor_cores:
        return ["encode_f32", "lse_merge"]
    import rank_latent_attention_b200 as flare
    return ["encode_tc"] + (["lse_merge"] if flare.flare_encode_splits(B, H, N) > 1 else [])


def mix_kernels(B: int, H: int, N: int, tensor_cores: bool = True) -> list:
    """The kernels of one flarepp_mix call: two encodes and the decode."""
    enc = encode_kernels(B, H, N, tensor_cores)
    return enc + enc + ["decode_tc" if tensor_cores else "decode_f32"]


def to_host(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def rms(x) -> float:
    return float(np.sqrt(np.mean(np.square(x))))


def stated_bound(want: np.ndarray, dtype: str) -> float:
    return TOL_F32_ABS if dtype == "f32" else TOL_BF16_REL_RMS * rms(want)


def _finite(name, got):
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"


def assert_stated(name: str, got: np.ndarray, want: np.ndarray, dtype: str):
    """The stated bar: fp32 1e-4 absolute; bf16 inputs 2e-2 x RMS(oracle)."""
    assert got.shape == want.shape, (name, got.shape, want.shape)
    _finite(name, got)
    err = float(np.max(np.abs(got - want)))
    b = stated_bound(want, dtype)
    assert err <= b, f"{name}: max|err| {err:.3e} > stated bound {b:.3e}"
    return err, b


def assert_bf16_storage(name: str, got: np.ndarray, want: np.ndarray, rows: np.ndarray, c: float):
    """Per-head bar of the bf16-storage path; arrays are [B, H, ...], rows [B, H, R, D]."""
    assert got.shape == want.shape, (name, got.shape, want.shape)
    _finite(name, got)
    atol = TOL_BF16_REL_RMS * rms(want)
    B, H = got.shape[:2]
    worst = 0.0
    for b in range(B):
        for h in range(H):
            err = float(np.max(np.abs(got[b, h] - want[b, h])))
            lim = atol + c * 2.0 ** -9 * float(np.max(np.abs(rows[b, h])))
            assert err <= lim, f"{name}[b={b},h={h}]: max|err| {err:.3e} > {lim:.3e}"
            worst = max(worst, err / lim)
    return worst


def assert_backward_bar(name: str, got: np.ndarray, want: np.ndarray, dtype: str, tensor_cores: bool):
    """The backward's bar; arrays are [B, H, ...] (dK, dV) or [H, ...] (d_seeds).

    The excess |g - r| - rel |r| (rel = 2^-8 covers the bf16 store of g, 0
    for fp32) must stay within
      CUDA-core kernels (fp32 arithmetic):  1e-4 x RMS(r)
      tensor-core kernels (bf16 operands):  2e-2 x RMS(r) + 16 x 2^-9 x max|r| of the head
    The tensor-core kernels round the softmax-gradient weights and the
    copies of dZ and dQ_dyn to bf16 (2^-9 relative each); a gradient sums
    such terms, so its error scales with the largest gradients of the head:
    on the heavy-tailed workload (tokens x8) max|dK| is 450 x RMS(dK), and
    the measured error is 1.4e-2 x max|dK| (7 x 2^-9).  It is the same form
    as the forward's bf16-storage bar (c = 16 for the decode output).
    """
    assert got.shape == want.shape, (name, got.shape, want.shape)
    _finite(name, got)
    rel = 0.0 if dtype == "f32" else 2.0 ** -8
    excess = np.abs(got - want) - rel * np.abs(want)
    r = rms(want)
    if not tensor_cores:
        worst = float(np.max(excess))
        assert worst <= 1e-4 * r, f"{name}: excess {worst:.3e} > {1e-4 * r:.3e}"
        return worst / max(r, 1e-30)
    lead = want.shape[:1] if want.ndim == 3 else want.shape[:2]
    worst = 0.0
    for idx in np.ndindex(*lead):
        lim = TOL_BF16_REL_RMS * r + 16 * 2.0 ** -9 * float(np.max(np.abs(want[idx])))
        e = float(np.max(excess[idx]))
        assert e <= lim, f"{name}{list(idx)}: excess {e:.3e} > {lim:.3e}"
        worst = max(worst, e / lim)
    return worst
