"""Derives the coefficients of the degree-3 polynomial that the kernels use
for 2^f on f in [-1/2, 1/2] (nea_device.cuh, exp2_poly2): a least-squares fit
of the relative error on a dense grid, reweighted (Lawson's iteration) until
the weighted fit approaches the minimax fit, then rounded to float32.

    python causal_gqa_attention_sm_b200/csrc/exp2_poly_fit.py

prints the four coefficients and the maximum relative error of the float32
Horner evaluation on the interval.  With range reduction x = j + f (j the
nearest integer) and 2^x = 2^j * p(f), the same relative error holds for
every x whose 2^x is a normal float32."""
import numpy as np


def fit(deg=3, iters=200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    w = np.ones_like(f)
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        W = w / y  # relative error
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        e = np.abs(V @ c - y) / y
        w = w * np.sqrt(e / e.max()) + 1e-12
        w /= w.sum()
    c32 = c.astype(np.float32)
    r = np.float32(c32[deg])
    f32 = f.astype(np.float32)
    for k in range(deg - 1, -1, -1):
        r = (r * f32 + c32[k]).astype(np.float32)
    return c32, float(np.max(np.abs(r.astype(np.float64) - y) / y))


if __name__ == "__main__":
    c, err = fit()
    print(" ".join(repr(float(v)) for v in c))
    print(f"max relative error {err:.3e}")
