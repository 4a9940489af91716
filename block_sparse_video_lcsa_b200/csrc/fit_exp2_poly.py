"""Fit the polynomial behind the attention kernel's FMA-pipe exponential.

2^x = 2^n * 2^f with n = round(x) and f in [-1/2, 1/2] (Cody and Waite's
argument reduction); 2^f is approximated by a degree-3 polynomial whose
relative error is minimised in the max norm by iteratively reweighted least
squares on a dense grid. Prints the fp32 coefficients that k3_attention_tc.cu
holds and the error of an fp32 Horner evaluation.

    python block_sparse_video_lcsa_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(deg=3, iters=200, grid=20001):
    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    w = np.ones_like(f)
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        A = V / y[:, None] * np.sqrt(w)[:, None]
        c, *_ = np.linalg.lstsq(A, np.sqrt(w), rcond=None)
        rel = (V @ c) / y - 1
        w = w * (1 + 50 * np.abs(rel) / np.abs(rel).max())
        w /= w.mean()
    return c.astype(np.float32)


def horner32(c, f):
    p = np.full(f.shape, c[-1], dtype=np.float32)
    for k in range(len(c) - 2, -1, -1):
        p = (p.astype(np.float64) * f + c[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    err = np.abs(horner32(c, f.astype(np.float64)) / np.exp2(f.astype(np.float64)) - 1).max()
    for k, v in enumerate(c):
        print("kExp2C%d = %.17gf" % (k, v))
    print("max relative error (fp32 Horner): %.3e" % err)
