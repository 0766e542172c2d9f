"""Coefficients of exp2_fma_x2 (msa_common.cuh): the degree-5 polynomial p with p(f) ~ 2^f on
[-1/2, 1/2], minimax in RELATIVE error, by the Remez exchange algorithm, rounded to fp32.

    python gen_exp2_poly.py      # prints the fp32 coefficients (c0 .. c5) as bit patterns

Method: start from Chebyshev extrema; each round solves p(x_i) - 2^x_i = (-1)^i E 2^x_i at the
deg + 2 reference points for the coefficients and the levelled error E, then moves the points to
the alternating extrema of the relative error on a fine grid. The fp32 Horner error is measured on
a grid of fp32 arguments.
"""
import numpy as np


def remez(deg=5, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    xs = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], xs) - np.exp2(xs)) / np.exp2(xs)
        d = np.diff(err)
        cand = np.concatenate(([0], np.where(np.sign(d[:-1]) != np.sign(d[1:]))[0] + 1, [len(xs) - 1]))
        sel = [cand[0]]
        for k in cand[1:]:
            if np.sign(err[k]) == np.sign(err[sel[-1]]):
                if abs(err[k]) > abs(err[sel[-1]]):
                    sel[-1] = k
            else:
                sel.append(k)
        while len(sel) > n:
            sel.pop(0 if abs(err[sel[0]]) < abs(err[sel[-1]]) else -1)
        if len(sel) < n:
            break
        x = xs[sel]
    return c


def fp32_coefficients(deg=5):
    return remez(deg).astype(np.float32)


def horner_fp32_rel_error(c32, a=-0.5, b=0.5, n=1000001):
    """Max relative error of the fp32 Horner evaluation of c32 against 2^f over fp32 f in [a, b]."""
    f = np.linspace(a, b, n).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float(np.abs((p.astype(np.float64) - ref) / ref).max())


if __name__ == "__main__":
    c = fp32_coefficients()
    print([hex(int(v.view(np.uint32))) for v in c], "fp32 Horner relative error", horner_fp32_rel_error(c))
