"""Fits the cubic used by the attention kernel's FMA-pipe exp2.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite
style range reduction; the kernel rounds with the 1.5 * 2^23 addition trick and
adds n to the float's exponent field).  2^f is approximated by
c0 + c1 f + c2 f^2 + c3 f^3, fitted here by least squares on the relative
error at Chebyshev nodes of [-1/2, 1/2], then refined by iteratively
reweighted least squares towards the minimax (equal-ripple) solution.  Prints
the coefficients (float32) and the maximum relative error on a dense grid.

    python blockwise_attn_ffn_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(degree=3, nodes=64, iters=30):
    k = np.arange(nodes)
    f = -0.5 * np.cos(np.pi * (k + 0.5) / nodes)          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]
    w = np.ones(nodes)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * w[:, None], w, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * (err / err.max()) ** 0.5 + 1e-12
        w /= w.max()
    return c.astype(np.float32)


def max_rel_err(c):
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float64)
    p = np.polyval(c[::-1].astype(np.float64), f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {v!r}")
    print("max relative error", max_rel_err(c))
