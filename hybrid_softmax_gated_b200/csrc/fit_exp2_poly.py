"""Fit the polynomial the attention kernel uses for part of its exponentials.

The softmax computes p = 2^x for x <= 8.  Most values go to the SFU
(ex2.approx); a fraction is computed on the FMA pipe instead, with the
classic range reduction of Cody and Waite: x = n + f with n = rint(x) and
f in [-1/2, 1/2], then 2^x = 2^n * P(f), where 2^n is added to the exponent
field of P(f).  P is a degree-3 polynomial close to the minimax one for the
relative error of 2^f on [-1/2, 1/2], obtained here by a Remez exchange.

    python hybrid_softmax_gated_b200/csrc/fit_exp2_poly.py

prints the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the maximum
relative error, measured in float32 Horner evaluation; the kernel's
constants are these numbers rounded to float32.  The error (~9e-5) is far
below the 2^-9 relative precision of the bf16 P that the next product uses.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    """Minimax polynomial for the relative error of 2^f on [LO, HI]."""
    n = deg + 2
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    xs = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_j c_j x^j - 2^x = (-1)^i E 2^x  (relative error equioscillation)
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        sgn = np.sign(err)
        idx = np.flatnonzero(np.diff(sgn) != 0)
        bounds = np.concatenate(([0], idx + 1, [len(grid)]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        xs = grid[ext]
    return c


def f32_horner_error(c):
    c32 = [np.float32(v) for v in c]
    f = np.linspace(LO, HI, 400001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for v in c32[-2::-1]:
        p = p * f + v
    exact = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - exact) / exact)), c32


if __name__ == "__main__":
    c = remez()
    e, c32 = f32_horner_error(c)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r}f  ({float(v).hex()})")
    print(f"max relative error (float32 Horner on [-1/2, 1/2]): {e:.3e}")
