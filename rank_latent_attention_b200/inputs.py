"""Seeded synthetic inputs for the FLARE++ mixer forward.

This module only draws random numbers.  It holds none of the mixer's arithmetic,
so both the CUDA path (through the binding) and the fp64 oracle can read the
same tensors without sharing any compute code.

Every tensor is drawn in float32 from a numpy ``Generator`` that is seeded per
(workload, tensor, batch, head) unit, then rounded once to the workload's
dtype (round-to-nearest-even for bf16).  Because each unit has its own seed,
any subset of heads can be regenerated on its own (the oracle checks sampled
heads of the million-token workload without drawing the other heads), and
the draw can run on a thread pool without changing a single value.

Workloads (shapes and value recipes of the pages' settings; no dataset is
used, these stand in for the PDE meshes and point clouds the pages train on):

==========  ====================================  =====  ==========================================
name        B, H, N, M, D                         dtype  values
==========  ====================================  =====  ==========================================
tiny_f32    2, 4, 1024, 32, 16                    f32    Q~, K, V ~ 0.5 * N(0,1)
cloud       8, 8, 972, 64, 16                     bf16   Q~, K, V ~ N(0,1)/sqrt(D); N % 128 != 0
mesh2d      4, 8, 11271 (221 x 51 grid), 128, 32  bf16   K, V: 8 random sinusoids over the grid
                                                         + 0.1 N(0,1); Q~ ~ N(0,1)/sqrt(D)
long        32, 8, 4096, 256, 32                  bf16   N(0,1)/sqrt(D); 1% outlier tokens x8
million     1, 16, 1048576, 256, 64               bf16   Q~, K, V ~ N(0,1)/sqrt(D)
==========  ====================================  =====  ==========================================

Layouts: ``seeds`` is [H][M][D] (one learned seed set per head, shared by the
batch); ``K`` and ``V`` are [B][H][N][D]; all row-major and contiguous.
"""
from __future__ import annotations

import concurrent.futures as _fut
import dataclasses
import math
import os

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_head", "make_seeds", "make_upstream", "custom"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    M: int
    D: int
    dtype: str  # "f32" or "bf16"
    kind: str  # value recipe: "gauss", "mesh", "outliers"
    index: int  # seed base: 1000 + index
    scale: float | None = None  # Gaussian std; None means 1/sqrt(D)
    grid: tuple[int, int] | None = None  # mesh2d grid (nx, ny), N = nx * ny
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0

    @property
    def std(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def flops(self) -> float:
        """Algorithmic FLOPs of one mixer forward: 3 steps x 2 GEMMs x 2*N*M*D per head."""
        return 12.0 * self.N * self.M * self.D * self.B * self.H

    def tokens(self) -> int:
        return self.B * self.N


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_f32", 2, 4, 1024, 32, 16, "f32", "gauss", 0, scale=0.5),
        Workload("cloud", 8, 8, 972, 64, 16, "bf16", "gauss", 1),
        Workload("mesh2d", 4, 8, 11271, 128, 32, "bf16", "mesh", 2, grid=(221, 51)),
        Workload("long", 32, 8, 4096, 256, 32, "bf16", "outliers", 3,
                 outlier_frac=0.01, outlier_gain=8.0),
        Workload("million", 1, 16, 1 << 20, 256, 64, "bf16", "gauss", 4),
    ]
}

_TENSOR_ID = {"seeds": 0, "K": 1, "V": 2, "outliers": 3, "mesh": 4, "dY": 5, "climb": 6}


def custom(B, H, N, M, D, dtype="bf16", kind="gauss", seed_index=99, scale=None) -> Workload:
    """An ad-hoc workload (edge-case tests): Gaussian values, given shapes."""
    return Workload(f"custom_{B}x{H}x{N}x{M}x{D}_{dtype}", B, H, N, M, D, dtype, kind,
                    seed_index, scale=scale)


def _rng(w: Workload, tensor: str, b: int = 0, h: int = 0) -> np.random.Generator:
    return np.random.default_rng([w.seed, _TENSOR_ID[tensor], b, h])


def _round(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the workload dtype, returned as float32 holding exact values."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype != "bf16":
        raise ValueError(f"unknown dtype {dtype!r}")
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # round-to-nearest-even on the upper 16 bits (inputs here are finite)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _outlier_rows(w: Workload, b: int) -> np.ndarray:
    """Token indices scaled by the outlier gain for batch element b (shared by all heads)."""
    count = int(math.floor(w.outlier_frac * w.N))
    return np.sort(_rng(w, "outliers", b).permutation(w.N)[:count])


def _mesh_field(w: Workload, b: int, h: int) -> tuple[np.ndarray, np.ndarray]:
    """K and V for one head of the mesh2d workload: per channel, 8 sinusoids over the grid."""
    nx, ny = w.grid
    assert nx * ny == w.N
    g = _rng(w, "mesh", b, h)
    x = (np.arange(nx, dtype=np.float64) / (nx - 1))[:, None].repeat(ny, 1).reshape(-1)
    y = (np.arange(ny, dtype=np.float64) / (ny - 1))[None, :].repeat(nx, 0).reshape(-1)
    out = []
    for _ in range(2):  # K then V
        f = np.zeros((w.N, w.D), dtype=np.float64)
        for d in range(w.D):
            for _k in range(8):
                a = g.normal(0.0, math.sqrt(1.0 / 8.0))
                while True:
                    fx, fy = int(g.integers(0, 5)), int(g.integers(0, 5))
                    if fx or fy:
                        break
                phi = g.uniform(0.0, 2.0 * math.pi)
                f[:, d] += a * np.sin(2.0 * math.pi * (fx * x + fy * y) + phi)
        f += 0.1 * g.standard_normal((w.N, w.D))
        out.append(f.astype(np.float32))
    return out[0], out[1]


def make_seeds(w: Workload) -> np.ndarray:
    """Latent seeds Q~ as float32 [H][M][D] holding values exact in the workload dtype."""
    s = np.empty((w.H, w.M, w.D), dtype=np.float32)
    for h in range(w.H):
        s[h] = _rng(w, "seeds", 0, h).standard_normal((w.M, w.D), dtype=np.float32) * np.float32(w.std)
    return _round(s, w.dtype)


def make_head(w: Workload, b: int, h: int) -> tuple[np.ndarray, np.ndarray]:
    """K and V of one (batch, head) unit as float32 [N][D], exact in the workload dtype."""
    if w.kind == "mesh":
        k, v = _mesh_field(w, b, h)
    else:
        k = _rng(w, "K", b, h).standard_normal((w.N, w.D), dtype=np.float32)
        v = _rng(w, "V", b, h).standard_normal((w.N, w.D), dtype=np.float32)
        k *= np.float32(w.std)
        v *= np.float32(w.std)
        if w.kind == "outliers":
            rows = _outlier_rows(w, b)
            k[rows] *= np.float32(w.outlier_gain)
            v[rows] *= np.float32(w.outlier_gain)
    return _round(k, w.dtype), _round(v, w.dtype)


def make_upstream(w: Workload) -> np.ndarray:
    """An upstream gradient dY [B,H,N,D] for the backward: N(0,1) values,
    float32 holding values exact in the workload dtype."""
    dY = np.empty((w.B, w.H, w.N, w.D), dtype=np.float32)
    for b in range(w.B):
        for h in range(w.H):
            dY[b, h] = _rng(w, "dY", b, h).standard_normal((w.N, w.D), dtype=np.float32)
    return _round(dY, w.dtype)


def make_climbing(H: int, N: int, M: int, D: int, jump_tile: int, seed_index: int = 131):
    """Encode inputs whose logits climb along the tokens (bf16, B = 1).

    Query m is e + Q~_m / 4 and key n is a_n e + K_n, with e a seeded unit
    vector and Q~, K, V a Gaussian workload's.  a_n = 6 t + 2 z_n for token n
    of 64-token tile t (z ~ N(0, 1)), plus 120 in tile jump_tile and minus 60
    in the tiles after it, so the logits of token n sit near a_n for every
    query.  Returns (Q [H,M,D], K [1,H,N,D], V [1,H,N,D]) as float32 holding
    bf16-exact values.
    """
    w = custom(1, H, N, M, D, dtype="bf16", seed_index=seed_index)
    seeds, K, V = make_inputs(w)
    g = _rng(w, "climb")
    e = g.standard_normal(D)
    e /= np.linalg.norm(e)
    tile = np.arange(N) // 64
    a = 6.0 * tile + 2.0 * g.standard_normal(N)
    a[tile == jump_tile] += 120.0
    a[tile > jump_tile] -= 60.0
    Q = e[None, None, :] + 0.25 * seeds.astype(np.float64)
    Kc = a[None, None, :, None] * e + K.astype(np.float64)
    return _round(Q.astype(np.float32), "bf16"), _round(Kc.astype(np.float32), "bf16"), V


def make_inputs(w: Workload, threads: int | None = None):
    """All inputs of a workload: (seeds [H,M,D], K [B,H,N,D], V [B,H,N,D]) as float32 arrays.

    Values are exactly representable in ``w.dtype``; callers convert to the
    device dtype without further rounding.
    """
    K = np.empty((w.B, w.H, w.N, w.D), dtype=np.float32)
    V = np.empty_like(K)

    def unit(bh):
        b, h = divmod(bh, w.H)
        K[b, h], V[b, h] = make_head(w, b, h)

    n = threads or min(32, os.cpu_count() or 1)
    if n > 1 and w.B * w.H > 1:
        with _fut.ThreadPoolExecutor(n) as ex:
            list(ex.map(unit, range(w.B * w.H)))
    else:
        for bh in range(w.B * w.H):
            unit(bh)
    return make_seeds(w), K, V
