"""Fit the polynomial that the kernels' software exp2 uses for 2^f, f in [-1/2, 1/2].

    python bwd_causal_sdpa_b200/csrc/fit_exp2_poly.py [degree]

Near-minimax fit of the relative error by iteratively reweighted least squares
(Lawson's algorithm) on a dense grid; the leading coefficient is pinned to 1 so
that 2^0 is exact. Prints the coefficients, rounded to float32, and the worst
relative error of the float32 Horner evaluation. The kernels split x = n + f
with n = round(x), evaluate this polynomial on the FMA pipe and add n to the
float's exponent field; the rest of the exponentials use the MUFU ex2 unit.
"""

import sys

import numpy as np


def fit(degree: int, iters: int = 200):
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5        # Chebyshev-spaced grid on [-1/2, 1/2]
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)[:, 1:]    # f, f^2, ..., f^deg (c0 = 1 fixed)
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w) / target                            # relative error weighting
        c, *_ = np.linalg.lstsq(V * sw[:, None], (target - 1.0) * sw, rcond=None)
        err = np.abs((1.0 + V @ c) / target - 1.0)
        w = w * (err + 1e-300)
        w /= w.sum()
    return np.concatenate([[1.0], c]).astype(np.float32)


def horner_f32(c, f):
    f = np.float32(f)
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = np.float32(p * f + np.float32(c[k]))
    return p


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = fit(deg)
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    p = horner_f32(c, f)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0).max()
    print("coefficients c0..c%d:" % deg, ", ".join("%.9ef" % x for x in c))
    print("max relative error (float32 Horner): %.3e" % rel)
