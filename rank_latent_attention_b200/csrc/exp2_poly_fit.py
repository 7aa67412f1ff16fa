"""Coefficients of the degree-3 polynomial that the softmax kernels use for
2^f on f in [-1/2, 1/2] (exp2_poly3 in common.cuh).

Minimax in the relative error max |p(f) / 2^f - 1|, found by the Remez
exchange algorithm: solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on n + 2 reference
points, move the references to the extrema of the weighted error, repeat.
The coefficients are then rounded to fp32, and the error of the fp32
evaluation (Horner with fused multiply-adds) is measured on a dense grid.

Run:  python exp2_poly_fit.py   (prints the coefficients and the error bound)
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree=DEGREE, lo=LO, hi=HI, iters=30):
    n = degree
    # Chebyshev extrema as the initial reference
    k = np.arange(n + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        y = np.exp2(x)
        # unknowns c_0..c_n, E:  sum c_j x^j - (-1)^i E y_i = y_i
        A = np.hstack([np.vander(x, n + 1, increasing=True), (-(-1.0) ** k * y)[:, None]])
        sol = np.linalg.solve(A, y)
        coef = sol[:-1]
        err = np.polyval(coef[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        sign = np.sign(err)
        breaks = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(grid.size), breaks)
        ext = np.array([r[np.argmax(np.abs(err[r]))] for r in runs])
        if ext.size < n + 2:
            break
        if ext.size > n + 2:  # keep the n + 2 largest, preserving alternation by trimming the ends
            while ext.size > n + 2:
                if abs(err[ext[0]]) < abs(err[ext[-1]]):
                    ext = ext[1:]
                else:
                    ext = ext[:-1]
        x = grid[ext]
    return coef


def fp32_eval(coef32, f):
    """Horner with fused multiply-adds in fp32 (product and sum exact in fp64, one rounding)."""
    f = f.astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c)).astype(np.float32)
    return p


def fit():
    coef = remez()
    coef32 = coef.astype(np.float32)
    f = np.linspace(LO, HI, 1 << 20).astype(np.float32)
    rel = np.abs(fp32_eval(coef32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    return coef32, float(rel.max())


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v):.9g}f  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error of the fp32 evaluation on [{LO}, {HI}]: {e:.3e}")
