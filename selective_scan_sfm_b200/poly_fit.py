"""Fits the minimax polynomials the kernels use on the FMA pipe, by the Remez exchange.

    python -m selective_scan_sfm_b200.poly_fit

* exp2(f) on f in [-1/2, 1/2], degree 5, minimising the maximum RELATIVE error.  With the
  Cody-Waite split x = j + f (j = round(x)), 2^x = 2^j * p(f); 2^j goes straight into
  the exponent field.  (W. J. Cody and W. Waite, "Software Manual for the Elementary
  Functions", 1980: argument reduction; the polynomial is fitted here.)
* log1p(w) / w on w in [0, 1], degree 7, minimising the maximum RELATIVE error, so that
  softplus(v) = max(v, 0) + w * q(w) with w = e^-|v| keeps its relative accuracy where
  w is small (softplus of very negative v).

Prints the coefficients (rounded to fp32) and the error of the fp32 Horner evaluation on
a dense grid; the values in csrc/sfm_device.cuh are this script's output.
"""
from __future__ import annotations

import numpy as np


def remez(g, lo, hi, deg, relative, iters=60):
    """Minimax polynomial (coefficients low -> high) of degree `deg` for g on [lo, hi]."""
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))  # Chebyshev extrema
    dense = np.linspace(lo, hi, 200001)
    E = 0.0
    c = np.zeros(deg + 1)
    for _ in range(iters):
        w = np.abs(g(x)) if relative else np.ones_like(x)
        A = np.vander(x, deg + 1, increasing=True)
        M = np.hstack([A, ((-1.0) ** k * w)[:, None]])
        sol = np.linalg.solve(M, g(x))
        c, E = sol[:-1], sol[-1]
        err = np.polynomial.polynomial.polyval(dense, c) - g(dense)
        if relative:
            err = err / np.abs(g(dense))
        # new reference: one extremum of the error per sign run
        s = np.sign(err)
        s[s == 0] = 1
        idx = np.flatnonzero(np.diff(s) != 0)
        bounds = np.concatenate([[0], idx + 1, [len(dense)]])
        ext = [a + np.argmax(np.abs(err[a:b])) for a, b in zip(bounds[:-1], bounds[1:])]
        if len(ext) < n:
            break
        while len(ext) > n:  # drop the smaller end extremum
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        newx = dense[ext]
        if np.allclose(newx, x, rtol=0, atol=1e-15):
            break
        x = newx
    return c, abs(E)


def horner_f32(c, x):
    x = x.astype(np.float32)
    cc = [np.float32(v) for v in c]
    p = np.full_like(x, cc[-1])
    for v in cc[-2::-1]:
        p = (p * x + v).astype(np.float32)  # the kernels use fused multiply-add; this bounds it
    return p.astype(np.float64)


def report():
    out = {}
    c, E = remez(np.exp2, -0.5, 0.5, 5, relative=True)
    f = np.linspace(-0.5, 0.5, 400001)
    e32 = np.max(np.abs(horner_f32(c, f) / np.exp2(f) - 1))
    out["exp2"] = (np.float32(c), E, e32)
    q = lambda w: np.where(w == 0, 1.0, np.log1p(w) / np.where(w == 0, 1.0, w))
    c2, E2 = remez(q, 0.0, 1.0, 7, relative=True)
    w = np.linspace(0.0, 1.0, 400001)
    e32b = np.max(np.abs(horner_f32(c2, w) / q(w) - 1))
    out["log1p_over_w"] = (np.float32(c2), E2, e32b)
    return out


if __name__ == "__main__":
    for name, (c, E, e32) in report().items():
        print("%s: minimax error %.3e, fp32 Horner error %.3e" % (name, E, e32))
        print("  " + ", ".join("%.9ef" % v for v in c))
