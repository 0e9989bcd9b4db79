"""Fit the cubic used by exp2_poly2() in sm100.cuh.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody-Waite range reduction); p is a degree-3 polynomial minimising the
maximum relative error of p(f) against 2^f on that interval, obtained here by
Lawson's iteratively re-weighted least squares. The coefficients are rounded
to fp32, as the kernel uses them.

    python mla_causal_attention_attn_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(deg: int = 3, iters: int = 400):
    f = np.linspace(-0.5, 0.5, 40001)
    y = np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True)
    wt = np.ones_like(f)
    c = None
    for _ in range(iters):
        W = wt / y
        c = np.linalg.lstsq(A * W[:, None], y * W, rcond=None)[0]
        err = np.abs(A @ c - y) / y
        wt = wt * err
        wt /= wt.sum()
    c32 = np.array([np.float32(x) for x in c], dtype=np.float64)
    rel = np.abs(A @ c32 - y) / y
    return [float(np.float32(x)) for x in c], float(rel.max())


if __name__ == "__main__":
    coeffs, err = fit()
    print("c0..c3 =", ", ".join(f"{c!r}f" for c in coeffs))
    print("max relative error on [-1/2, 1/2]:", err)
