"""Fit the cubic used by the attention kernel's FMA-pipe exp2.

exp2(x) is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2].
2^f is approximated by c0 + c1 f + c2 f^2 + c3 f^3, fitted here by least
squares of the RELATIVE error on Chebyshev nodes of [-1/2, 1/2] (close to the
minimax fit), in float64, then rounded to float32.  The attention kernel
rounds every probability to bf16 (8 significant bits) before the PV product,
so a relative error near 1e-4 is far below what that rounding adds.

    python fit_exp2_poly.py      # prints the coefficients and the max error

The kernel's constants are this script's output.
"""

import numpy as np


def fit(degree=3, nodes=4001):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes in [-1/2, 1/2]
    target = np.exp2(f)
    # minimise sum((p(f) - 2^f) / 2^f)^2: divide each row by 2^f
    A = np.stack([f ** i for i in range(degree + 1)], axis=1) / target[:, None]
    coef, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return coef


def max_rel_error(coef32):
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(f)
    for c in coef32[::-1]:
        p = p * f + float(c)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit().astype(np.float32)
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r:>24}  ({float(v).hex()})")
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c):.3e}")
