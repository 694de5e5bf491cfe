"""Fits the polynomial that the attention kernel uses for part of its
exponentials: 2^f on f in [-1/2, 1/2], degree 3, minimising the maximum
relative error.

Method: Lawson's algorithm (iteratively reweighted least squares converging
to the minimax fit) on a dense grid, then a check of the float32 Horner
evaluation.  The kernel combines it with the range reduction
2^x = 2^n * 2^f, n = round(x), f = x - n.

    python fit_exp2_poly.py      # prints the coefficients and the error
"""

import numpy as np


def fit(degree=3, points=20001, iterations=300):
    f = np.linspace(-0.5, 0.5, points)
    y = 2.0 ** f
    vander = np.vander(f, degree + 1, increasing=True)
    w = np.full(points, 1.0 / points)
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(vander / y[:, None] * sw[:, None], sw, rcond=None)
        err = np.abs(vander @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    return c


def horner_f32(c, f):
    c32 = c.astype(np.float32)
    f32 = f.astype(np.float32)
    p = np.full_like(f32, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = p * f32 + c32[k]
    return p


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(horner_f32(c, f).astype(np.float64) / 2.0 ** f - 1.0).max()
    for k, v in enumerate(c.astype(np.float32)):
        print(f"c{k} = {float(v):.9g}f")
    print(f"max relative error (float32 Horner) = {rel:.3g}")
