"""Fit the cubic used by exp2_fma() in sm100.cuh.

2^x = 2^n * 2^f with n = round(x) and f in [-1/2, 1/2].  The cubic p(f) is
fitted for minimum maximum relative error |p(f)/2^f - 1| on [-1/2, 1/2] by
iteratively reweighted least squares on a Chebyshev grid (a Lawson-style
approximation of the minimax fit), then rounded to fp32.  Running this file
prints the coefficients (lowest order first) and the maximum relative error of
the fp32 Horner evaluation, which is what the kernel computes.
"""
from __future__ import annotations

import numpy as np


def fit(deg: int = 3, iters: int = 60):
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True) / y[:, None]
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * w[:, None], w, rcond=None)
        err = V @ c - 1.0
        w = w * (1.0 + 4.0 * np.abs(err) / np.abs(err).max())
        w /= w.mean()
    return c.astype(np.float32)


def max_rel_error(coeffs, n: int = 200001) -> float:
    """Max relative error of the fp32 Horner evaluation on [-1/2, 1/2]."""
    c = np.asarray(coeffs, dtype=np.float32)
    ff = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.full_like(ff, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * ff + c[k]).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1.0).max())


if __name__ == "__main__":
    c = fit()
    print([float(x) for x in c], max_rel_error(c))
