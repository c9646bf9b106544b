"""Fit of the degree-4 polynomial p(r) ~ 2^r on [-1/2, 1/2] used by exp2_poly2 (ptx.cuh).

Weighted least squares of the relative error at Chebyshev nodes, refined by Lawson
reweighting towards the minimax (equioscillating) fit; then the coefficients are rounded
to fp32 and the fp32 Horner evaluation is checked against float64 2^r.

    python fit_exp2_poly.py        # prints the coefficients and the max relative error
"""
import numpy as np

DEG = 4


def fit(deg: int = DEG, iters: int = 60) -> np.ndarray:
    k = np.arange(4000)
    r = 0.5 * np.cos(np.pi * (k + 0.5) / len(k))
    y = np.exp2(r)
    A = np.vander(r, deg + 1, increasing=True) / y[:, None]
    b = np.ones_like(r)
    w = np.ones_like(r)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * np.sqrt(w)[:, None], b * np.sqrt(w), rcond=None)
        e = np.abs(A @ c - b)
        w = w * (e + 1e-30)
        w /= w.sum()
    return c


def horner_fp32(c: np.ndarray, r: np.ndarray) -> np.ndarray:
    c32 = c.astype(np.float32)
    p = np.full_like(r, c32[-1], dtype=np.float32)
    for ci in c32[-2::-1]:
        p = (p.astype(np.float64) * r + ci).astype(np.float32)   # one rounding per step, as an FMA
    return p


def max_rel_error(c: np.ndarray) -> float:
    r = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    return float(np.max(np.abs(horner_fp32(c, r).astype(np.float64) / np.exp2(r.astype(np.float64)) - 1)))


if __name__ == "__main__":
    c = fit()
    print("coefficients (r^0 .. r^4):", [repr(float(np.float32(x))) for x in c])
    print("max relative error (fp32 Horner): %.3e" % max_rel_error(c))
