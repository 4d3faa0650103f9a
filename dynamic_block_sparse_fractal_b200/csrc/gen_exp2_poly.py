"""Fits the polynomial used for exp2 on the FMA pipe (see exp2_poly.cuh).

Method: range reduction x = n + f with n = round(x), f in [-1/2, 1/2], so
2^x = 2^n * 2^f; 2^f is approximated by a polynomial p(f) whose coefficients
are chosen to minimise the maximum relative error |p(f) / 2^f - 1| on
[-1/2, 1/2] (Remez exchange, started from Chebyshev interpolation). 2^n is
applied by adding n to the float's exponent field.

    python gen_exp2_poly.py [degree]    # prints coefficients and max rel error
"""
import sys

import numpy as np


def remez_rel(deg, lo=-0.5, hi=0.5, iters=30):
    # start: interpolation at Chebyshev nodes
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (2 * k + 1) / (2 * (deg + 2)))
    x = np.sort(x)
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (equioscillating relative error)
        A = np.vander(x, deg + 1, increasing=True)
        sgn = (-1.0) ** np.arange(deg + 2)
        M = np.hstack([A, -(sgn * 2.0 ** x)[:, None]])
        sol = np.linalg.solve(M, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] >= err[i - 1] and err[i] >= err[i + 1]) or (err[i] <= err[i - 1] and err[i] <= err[i + 1]):
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        ecand = err[idx]
        # keep deg+2 alternating extrema of largest magnitude
        pts = [(cand[0], ecand[0])]
        for xx, ee in zip(cand[1:], ecand[1:]):
            if np.sign(ee) == np.sign(pts[-1][1]):
                if abs(ee) > abs(pts[-1][1]):
                    pts[-1] = (xx, ee)
            else:
                pts.append((xx, ee))
        while len(pts) > deg + 2:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < deg + 2:
            break
        x = np.array([p[0] for p in pts])
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_rel(deg)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001)
    e32 = np.abs(np.polyval(c32.astype(np.float64)[::-1], g) / 2.0 ** g - 1).max()
    print(f"degree {deg}: max rel error {e:.3e} (coefficients rounded to fp32: {e32:.3e})")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v):.9e}f")
