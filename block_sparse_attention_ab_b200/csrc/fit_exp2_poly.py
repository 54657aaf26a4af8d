"""Derive the coefficients of the degree-3 polynomial p(f) ~ 2^f on [-1/2, 1/2] used by
the attention kernel's software exp2 (Cody-Waite split 2^x = 2^round(x) * 2^f).

Method: relative-error weighted least squares on 4001 Chebyshev nodes, refined by
Lawson's iteratively reweighted least squares toward the minimax (equioscillating)
relative error. Prints the coefficients (fp32) and the achieved max relative error.
"""
import numpy as np


def fit(degree=3, nodes=4001, lawson_iters=200):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error system
    b = np.ones_like(f)
    w = np.ones_like(f) / nodes
    for _ in range(lawson_iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    fine = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(c32[::-1].astype(np.float64), fine)
    return c32, np.max(np.abs(p / np.exp2(fine) - 1))


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  /* 0x{np.float32(v).view(np.uint32):08x} */")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
