"""Fits the polynomial behind the FMA-pipe exp2 used by the attention softmax (exp2_poly2 in
fpx_sm100.cuh) and prints its coefficients and error bound.

Method: Cody-Waite style range reduction x = n + f with n = round(x), |f| <= 1/2, so that
2^x = 2^n * 2^f; 2^n is applied by adding n to the exponent field.  2^f on [-1/2, 1/2] is a
degree-3 polynomial whose coefficients minimise the maximum *relative* error, found with the
Remez exchange algorithm (equioscillation on 5 alternation points).  The coefficients are then
rounded to fp32 and the final error is measured on a dense grid.

    python dynamic_block_sparse_pooled_b200/csrc/exp2_poly_fit.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve  sum_j c_j x_i^j - 2^x_i = (-1)^i E 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        b = 2.0 ** x
        sol = np.linalg.solve(A, b)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new alternation points: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        if len(idx) >= n:
            # keep the n points with alternating signs and largest magnitude
            pts = []
            for i in idx:
                if not pts or np.sign(err[i]) != np.sign(err[pts[-1]]):
                    pts.append(i)
                elif abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            while len(pts) > n:
                if abs(err[pts[0]]) < abs(err[pts[-1]]):
                    pts.pop(0)
                else:
                    pts.pop()
            if len(pts) == n:
                x = grid[pts]
    return c


if __name__ == "__main__":
    c = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 1000001)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * grid.astype(np.float32) + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) - 2.0 ** grid) / 2.0 ** grid
    for k, v in enumerate(c32):
        print(f"C{k} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2] with fp32 coefficients: {rel.max():.3e}")
