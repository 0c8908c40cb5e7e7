"""Fit of the cubic that the prefill softmax uses for part of its 2^x.

Method (Cody-Waite style argument split, polynomial fitted here): for
x <= 0 in log2 units, n = round(x) and f = x - n in [-0.5, 0.5], so
2^x = 2^n * 2^f; 2^f is replaced by a cubic c0 + c1 f + c2 f^2 + c3 f^3 whose
coefficients minimise the maximum RELATIVE error over [-0.5, 0.5]
(iteratively reweighted least squares on a dense grid, a discrete stand-in
for a Remez exchange), then rounded to float32.  2^n is applied by adding n to
the float's exponent field.  The kernel rounds the result to bf16 (relative
spacing 2^-8), so a relative error below 1e-4 is invisible there.

``python -m attention_yarn_rope_b200.exp2_poly`` prints the coefficients and
the achieved error; ``csrc/sm100_ptx.cuh`` holds the same four numbers.
"""

from __future__ import annotations

import numpy as np


def fit(degree: int = 3, iters: int = 200, points: int = 20001):
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    A = np.vstack([f ** k for k in range(degree + 1)]).T / y[:, None]
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * w[:, None], w, rcond=None)
        rel = np.abs(A @ c - 1.0)
        w = w * (1.0 + 20.0 * rel / rel.max())
        w /= w.mean()
    return np.asarray(c, np.float32)


def max_rel_error(coeffs, points: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, points)
    p = np.polyval(np.asarray(coeffs, np.float64)[::-1], f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0..c3):", ", ".join(repr(float(x)) + "f" for x in c))
    print("max relative error:", max_rel_error(c))
