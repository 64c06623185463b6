"""Fits the polynomial that window_tc.cu uses for part of its exp2 evaluations.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (range reduction
in the manner of Cody and Waite); 2^f is approximated by a degree-3
polynomial whose maximum relative error on [-1/2, 1/2] is driven towards the
minimax value with Lawson's iteratively reweighted least squares. The softmax
weights that use it are rounded to bf16 right after (relative step 2^-8), so
a relative error near 1e-4 is far below what the result keeps.

Run: python exp2_poly_fit.py   (prints the float32 coefficients and the error
of the float32 Horner evaluation the kernel performs).
"""

import numpy as np


def fit(degree=3, iters=200, npts=4001):
    f = np.cos(np.linspace(0.0, np.pi, npts)) * 0.5  # Chebyshev-spaced on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f) / npts
    for _ in range(iters):
        sw = np.sqrt(w) / y  # relative error weighting
        c, *_ = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * err
        w /= w.sum()
    return c


def device_eval(c32, x):
    """float32 emulation of the kernel's evaluation order."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * f + np.float32(c32[k])).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    xs = np.linspace(-30.0, 8.0, 2000001).astype(np.float32)
    rel = np.abs(device_eval(c32, xs).astype(np.float64) - np.exp2(xs.astype(np.float64))) / np.exp2(
        xs.astype(np.float64))
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v):.9e}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error of the float32 evaluation on [-30, 8]: {rel.max():.3e}")
