"""Derives the coefficients kP0..kP3 of the FMA-pipe 2^f polynomial in
attn_spatial_sm100.cu (and prints its maximum relative error).

Method: Remez exchange for the degree-3 polynomial p that minimises
max |p(f) / 2^f - 1| over f in [-1/2, 1/2] (relative error, because the
softmax's exponentials are compared with each other, not with a fixed scale).
Start from the Chebyshev extrema, solve for the coefficients and the levelled
error E on the n + 2 reference points, move the reference to the alternating
extrema of the new error curve, repeat until the reference stops moving.  The
coefficients are then rounded to fp32, as the kernel stores them, and the
error is re-measured with the rounded values.

Run: python sequence_parallelism_st_b200/csrc/fit_exp2_poly.py
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def alternating_extrema(err):
    """Indices of the local extrema of err (ends included), one per sign run."""
    k = np.arange(1, err.size - 1)
    inner = k[(err[k] - err[k - 1]) * (err[k + 1] - err[k]) <= 0]
    pts = []
    for i in np.concatenate([[0], inner, [err.size - 1]]):
        if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
            if abs(err[i]) > abs(err[pts[-1]]):
                pts[-1] = i
        else:
            pts.append(int(i))
    return pts


def remez(n=DEGREE, lo=LO, hi=HI, iters=40, grid=400_001):
    g = np.linspace(lo, hi, grid)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n + 2)[::-1] / (n + 1))
    for _ in range(iters):
        # p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}  (levelled relative error)
        A = np.zeros((n + 2, n + 2))
        A[:, :n + 1] = x[:, None] ** np.arange(n + 1)[None, :]
        A[:, n + 1] = -((-1.0) ** np.arange(n + 2)) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:n + 1]
        err = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
        pts = alternating_extrema(err)
        while len(pts) > n + 2:              # keep the n + 2 largest, still alternating
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        if len(pts) < n + 2:
            break
        new_x = g[pts]
        if np.allclose(new_x, x, atol=1e-12):
            break
        x = new_x
    return c


if __name__ == "__main__":
    c = remez().astype(np.float32).astype(np.float64)
    f = np.linspace(LO, HI, 2_000_001)
    e = np.abs(np.polyval(c[::-1], f) / np.exp2(f) - 1.0).max()
    for i, v in enumerate(c):
        print(f"kP{i} = {float(np.float32(v))!r}f")
    print(f"max relative error on [{LO}, {HI}] with fp32 coefficients: {e:.4e}")
