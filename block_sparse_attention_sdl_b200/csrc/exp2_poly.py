"""Coefficients of the FMA-pipe exp2 used by the attention softmax.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by a cubic c0 + f (c1 + f (c2 + f c3)).  The cubic is the least-
squares fit, in relative error, of 2^f at 4096 Chebyshev nodes of [-1/2, 1/2]
(numpy.linalg.lstsq on the weighted Vandermonde system).  Its largest relative
error on the interval is printed; it must stay far below bf16's 2^-9 rounding
step, since the weights are rounded to bf16 right after.

Run: python exp2_poly.py  (prints the constants written into attn_km.cu).
"""
import numpy as np


def fit(degree=3, n=4096):
    k = np.arange(n)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * n))  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return c


def max_rel_error(c32, n=200001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.float32(c32[3])
    for ci in (c32[2], c32[1], c32[0]):
        p = (p * f + np.float32(ci)).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = [np.float32(x) for x in c]
    for i, x in enumerate(c32):
        print(f"c{i} = {float(x).hex()}  ({x!r})")
    print("max relative error:", max_rel_error(c32))
