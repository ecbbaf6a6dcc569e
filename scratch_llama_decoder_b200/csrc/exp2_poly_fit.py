"""Coefficients of the polynomial 2^f of exp2_poly2 (tcgen05.cuh).

The degree-3 polynomial p that minimises max |p(f) / 2^f - 1| over
f in [-1/2, 1/2], by the Remez exchange algorithm on a dense grid, rounded to
float32.  Run as a script it prints the four coefficients (lowest degree
first) and the maximum relative error of the float32 Horner evaluation.
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(deg=DEGREE, lo=LO, hi=HI, iters=40, grid=200001):
    """Minimax (relative error) polynomial coefficients, lowest degree first."""
    n = deg + 2
    # start from the Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    g = np.linspace(lo, hi, grid)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the n reference points
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            a[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(a, np.exp2(x))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
        # next reference: the extremum of each run of equal sign
        cuts = np.concatenate(([0], np.where(np.diff(np.sign(err)) != 0)[0] + 1, [grid]))
        ref = [k0 + int(np.argmax(np.abs(err[k0:k1]))) for k0, k1 in zip(cuts[:-1], cuts[1:])]
        if len(ref) != n:
            break
        x = g[ref]
    return c


def coefficients():
    """The float32 coefficients, lowest degree first."""
    return [float(v) for v in remez().astype(np.float32)]


def horner_rel_error(c32, points=100001):
    """Max relative error of the float32 Horner evaluation on [LO, HI]."""
    f = np.linspace(LO, HI, points).astype(np.float32)
    p = np.float32(c32[-1])
    for ck in c32[-2::-1]:
        p = (p * f + np.float32(ck)).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0).max())


if __name__ == "__main__":
    c = coefficients()
    for k, v in enumerate(c):
        print(f"C{k} = {v!r}f")
    print(f"max relative error (float32 Horner): {horner_rel_error(c):.3e}")
