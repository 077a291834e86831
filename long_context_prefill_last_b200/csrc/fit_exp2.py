"""Minimax polynomials for 2**f on f in [-1/2, 1/2] (relative error), by the
Remez exchange algorithm, for the FMA-pipe exp2 in ptx.cuh (exp2_poly3 /
exp2_poly5). Run to print the coefficients and their float32 error:

    python long_context_prefill_last_b200/csrc/fit_exp2.py

Method: 2**x = 2**n * 2**f with n = round(x), f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction); 2**f by a polynomial whose maximum
relative error on the interval is equioscillating (Remez, 1934).
"""
import numpy as np


def remez_relative(deg, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    xs = (lo + hi) / 2 + (hi - lo) / 2 * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve sum c_j x^j - f(x) = (-1)^i E f(x) at the reference
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x)
        sol = np.linalg.solve(A, f(xs))
        c, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of err
        idx = np.nonzero(np.diff(np.sign(np.diff(err))))[0] + 1
        cand = np.concatenate(([0], idx, [len(grid) - 1]))
        if len(cand) < n:
            break
        # keep n points with the largest |err| that alternate in sign
        pts = list(cand)
        while len(pts) > n:
            vals = np.abs(err[pts])
            j = int(np.argmin(vals))
            pts.pop(j)
        xs = grid[pts]
    return c, float(np.max(np.abs(err)))


def f32_error(c):
    """Max relative error of the float32 Horner evaluation over [-1/2, 1/2]."""
    x = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    c32 = [np.float32(v) for v in c]
    p = np.full_like(x, c32[-1])
    for v in reversed(c32[:-1]):
        p = (p * x + v).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    for deg in (3, 5):
        c, e = remez_relative(deg)
        print(f"degree {deg}: minimax rel error {e:.3e}, float32 Horner {f32_error(c):.3e}")
        print("  coefficients (c0..c%d): " % deg + ", ".join(f"{float(np.float32(v)):.9g}f" for v in c))
