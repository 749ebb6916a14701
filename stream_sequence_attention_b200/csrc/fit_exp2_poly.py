"""Derive the cubic used by the attention kernel to evaluate 2^f on the FMA
pipe for f in [-1/2, 1/2] (after rounding x to the nearest integer n,
2^x = 2^n * 2^f).  Weighted least squares on the relative error, re-weighted
(Lawson's iteration) towards the minimax solution; prints float32
coefficients c0..c3 and the float32-Horner maximum relative error
(about 7.5e-5, far below the bf16 rounding of P, 2^-9).

    python stream_sequence_attention_b200/csrc/fit_exp2_poly.py
"""

import numpy as np


def fit(deg=3, iters=200):
    f = np.linspace(-0.5, 0.5, 200001)
    y = 2.0 ** f
    w = np.ones_like(f)
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * (w / y)[:, None], w, rcond=None)
        err = (V @ c) / y - 1
        w = w * np.sqrt(np.abs(err) + 1e-30)
        w /= w.mean()
    c32 = c.astype(np.float32)
    x = f.astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * x + c32[k]).astype(np.float32)
    return c32, float(np.abs(p.astype(np.float64) / y - 1).max())


if __name__ == "__main__":
    c, e = fit()
    print("coefficients:", ", ".join(f"{v:.9g}f" for v in c))
    print("max relative error:", e)
