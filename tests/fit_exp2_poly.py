"""Fit the coefficients of the FMA-pipe 2^f used by the softmax (exp2_fma_pair in sm100_ptx.cuh).

p(f) = 1 + f * (c1 + f * (c2 + f * c3)) on f in [-1/2, 1/2], minimising the largest relative error
|p(f) / 2^f - 1| with Lawson's iteratively re-weighted least squares (a minimax fit). The constant
term is pinned to exactly 1, so that p(0) = 1 and the exponent trick maps x = -127 to +0 exactly.

Run: python tests/fit_exp2_poly.py   (prints the three fp32 coefficients and the fp32 error bound).
"""
import numpy as np


def fit(deg: int = 3, n: int = 4001, iters: int = 400):
    f = np.cos(np.linspace(0.0, np.pi, n)) * 0.5  # Chebyshev-spaced points on [-1/2, 1/2]
    y = np.exp2(f)
    # relative error r = (1 + sum c_k f^k) / y - 1  ->  sum c_k f^k / y = (y - 1) / y + r
    A = np.stack([f ** k / y for k in range(1, deg + 1)], axis=1)
    b = (y - 1.0) / y
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * r
        w /= w.sum()
    return c


def fp32_eval(c, f):
    """Horner in fp32 with one rounding per fused step (as fma.rn.f32x2 does)."""
    c = [np.float32(v) for v in c]
    f64 = f.astype(np.float64)
    p = np.float32(c[-1])
    for ck in reversed(c[:-1]):
        p = (p.astype(np.float64) * f64 + np.float64(ck)).astype(np.float32)
    return (p.astype(np.float64) * f64 + 1.0).astype(np.float32)


if __name__ == "__main__":
    c = fit()
    c32 = [float(np.float32(v)) for v in c]
    f = (np.linspace(-0.5, 0.5, 200001)).astype(np.float32)
    err = np.abs(fp32_eval(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0).max()
    for k, v in enumerate(c32, start=1):
        print(f"c{k} = {v!r}  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error in fp32: {err:.3e}")
