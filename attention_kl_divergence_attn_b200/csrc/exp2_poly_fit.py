"""Fits the polynomials that approximate 2**f on [-1/2, 1/2] used by exp2_fma().

Method: 2**x = 2**n * 2**f with n = rint(x) and f = x - n in [-1/2, 1/2]
(exact range reduction, no rounding error); 2**f is approximated by a
polynomial whose coefficients minimise the maximum relative error on
[-1/2, 1/2], found by iteratively re-weighted least squares on 4001 points
(Lawson's algorithm, which converges to the minimax solution).  The fitted
coefficients are rounded to fp32 and the achieved error is re-measured with
fp32 Horner evaluation.  Run: python exp2_poly_fit.py
"""
import numpy as np


def fit(deg, iters=200):
    f = np.linspace(-0.5, 0.5, 4001)
    y = 2.0 ** f
    V = np.vander(f, deg + 1, increasing=True) / y[:, None]   # relative error system
    w = np.ones_like(f) / f.size
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones_like(f) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    # fp32 Horner evaluation error
    p = np.float32(c32[-1])
    ff = f.astype(np.float32)
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    rel = np.max(np.abs(p.astype(np.float64) / y - 1.0))
    return c32, rel


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c, rel = fit(deg)
        print(f"degree {deg}: max relative error {rel:.3e}")
        print("  coefficients (c0..c%d):" % deg, ", ".join(f"{float(v):.9e}f" for v in c))
