"""Derives the degree-3 polynomial for 2^f, f in [-1/2, 1/2], used by the
kernel's FMA-pipe exp2 (exp2_poly2 in sm100.cuh).

Method: iteratively re-weighted least squares on a dense grid, minimising the
maximum relative error (a discrete minimax fit); the float32 coefficients are
then checked with float32 Horner evaluation. Prints the coefficients c0..c3
and the achieved max relative error (about 7.6e-5).
"""

import numpy as np


def fit(deg: int = 3, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = 2.0 ** f
    V = np.vander(f, deg + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq((V / y[:, None]) * w[:, None], w, rcond=None)
        err = (V @ c) / y - 1
        w = w * (np.abs(err) / np.abs(err).max()) ** 0.5 + 1e-3
    c32 = c.astype(np.float32)
    return c32, horner_f32(c32, f.astype(np.float32)) / y - 1


def horner_f32(c32, x32):
    acc = np.float32(c32[-1]) * np.ones_like(x32)
    for k in range(len(c32) - 2, -1, -1):
        acc = (acc * x32 + c32[k]).astype(np.float32)
    return acc


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", [float(v) for v in c])
    print("max relative error:", float(np.abs(err).max()))
