"""Fits the polynomial used by the kernels' FMA-pipe exp2 (attn_tc.cu).

2^x is split as 2^k * 2^f with k = round(x) and f = x - k in [-1/2, 1/2].
2^f is approximated by p(f) = c0 + c1 f + c2 f^2 + c3 f^3 (three FMAs in
Horner form), with c0..c3 minimising the maximum relative error
|p(f)/2^f - 1| on [-1/2, 1/2]: a Remez exchange on the relative error,
started from a least-squares fit on Chebyshev nodes.  The coefficients are
rounded to fp32 and the resulting error is reported.
Run: python fit_exp2_poly.py
"""
import numpy as np

DEG = 3


def poly(c, f):
    p = np.zeros_like(f) + c[-1]
    for k in range(len(c) - 2, -1, -1):
        p = p * f + c[k]
    return p


def rel_err(c, f):
    return poly(c, f) / np.exp2(f) - 1.0


def fit(iters=40):
    n = 400
    f = 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)
    w = 1.0 / np.exp2(f)
    A = np.stack([w * f ** k for k in range(DEG + 1)], 1)
    c = np.linalg.lstsq(A, np.ones(n), rcond=None)[0]
    grid = np.linspace(-0.5, 0.5, 400001)
    for _ in range(iters):
        e = rel_err(c, grid)
        cuts = np.nonzero(np.diff(np.sign(e)))[0]
        segs = np.split(np.arange(grid.size), cuts + 1)
        ext = np.array([seg[np.argmax(np.abs(e[seg]))] for seg in segs])
        if ext.size < DEG + 2:
            break
        # keep DEG+2 alternating extrema, largest first
        while ext.size > DEG + 2:
            ends = [0, ext.size - 1]
            drop = ends[int(np.argmin(np.abs(e[ext[ends]])))]
            ext = np.delete(ext, drop)
        x = grid[ext]
        M = np.zeros((DEG + 2, DEG + 2))
        for i, xi in enumerate(x):
            wi = 1.0 / np.exp2(xi)
            M[i, : DEG + 1] = [wi * xi ** k for k in range(DEG + 1)]
            M[i, DEG + 1] = -((-1) ** i)
        sol = np.linalg.solve(M, np.ones(DEG + 2))
        c = sol[: DEG + 1]
    return c


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 1000001)
    print("coefficients c0..c3 (fp32):", [repr(float(x)) for x in c32])
    print("max relative error: %.3e" % np.abs(rel_err(c32.astype(np.float64), g)).max())
