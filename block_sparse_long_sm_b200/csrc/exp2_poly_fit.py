"""Coefficients of the polynomial 2^x used for part of the softmax exponentials.

Method (Cody-Waite range reduction with a polynomial core): for x in
[-126, 127], write x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2];
then 2^x = 2^n * 2^f, where 2^n is added to the exponent field of the float
p(f) ~ 2^f.  p is the degree-3 polynomial that minimises the maximum
*relative* error on [-1/2, 1/2], found here by iteratively reweighted least
squares on a dense grid (a discrete Remez / Lawson iteration).  The result is
good to about 1e-4 relative error, below the 2^-9 rounding of the bf16
probabilities it feeds.

Run ``python exp2_poly_fit.py`` to print the coefficients pasted into
``attn.cuh`` (kExp2C0..kExp2C3) and the achieved error.
"""

import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        A = V / target[:, None] * np.sqrt(w)[:, None]
        b = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A, b, rcond=None)
        rel = np.abs(V @ c / target - 1.0)
        w = w * (rel + 1e-12)
        w /= w.mean()
    rel = np.abs(V @ c / target - 1.0)
    return c, float(rel.max())


def eval_fp32(x: np.ndarray, c) -> np.ndarray:
    """The kernel's arithmetic, step by step in fp32 (for the CPU check)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)                 # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n_bits = t.view(np.int32)
    xr = (t - magic).astype(np.float32)
    f = (x - xr).astype(np.float32)
    c = [np.float32(v) for v in c]
    p = np.float32(c[3])
    p = (p * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    out = (p.view(np.int32) + (n_bits << 23)).view(np.float32)
    return out


if __name__ == "__main__":
    c, err = fit()
    for i, v in enumerate(c):
        print(f"kExp2C{i} = {float(np.float32(v)):.9g}f")
    print("max relative error on [-0.5, 0.5]:", err)
