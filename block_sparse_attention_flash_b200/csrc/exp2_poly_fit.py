"""Fit the polynomial the attention softmax uses for part of its exp2 work.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction).  2^f is approximated by the degree-3
polynomial p(f) = c0 + c1 f + c2 f^2 + c3 f^3 that minimises the maximum
RELATIVE error on [-1/2, 1/2] (Remez exchange algorithm: alternate between
solving for coefficients that equioscillate on a reference set and moving
the reference to the extrema of the error).  The kernel rebuilds 2^n by
adding n to the exponent field of p(f).

Run `python exp2_poly_fit.py` to print the coefficients pasted into
sa_attn_fwd.cuh and the error bound the tests check.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # Chebyshev extrema as the first reference
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E * 2^x_i   (relative equioscillation)
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        new_ref = []
        start = 0
        for j in range(1, grid.size):
            if sign[j] != sign[j - 1]:
                seg = slice(start, j)
                new_ref.append(grid[seg][np.argmax(np.abs(err[seg]))])
                start = j
        seg = slice(start, grid.size)
        new_ref.append(grid[seg][np.argmax(np.abs(err[seg]))])
        if len(new_ref) != n:
            break
        ref = np.array(new_ref)
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.12e})")
    print(f"max relative error (exact arithmetic): {e:.3e}")
