"""Fits the cubic that the tcgen05 prefill kernel uses for 2^f, f in [-0.5, 0.5].

Remez exchange on the relative error (p(f) - 2^f) / 2^f, in float64; prints the
coefficients rounded to float32 and the resulting maximum relative error.
`python fit_exp2_poly.py` reproduces kExp2C0..kExp2C3 in prefill_tc.cuh.
"""
import numpy as np


def remez(n: int, a: float = -0.5, b: float = 0.5, iters: int = 30):
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))  # Chebyshev start
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, :n + 1] = xi ** np.arange(n + 1) / 2.0 ** xi
            A[i, n + 1] = (-1) ** i
        c = np.linalg.solve(A, np.ones(n + 2))[:n + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1
        segs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segs]
        if len(ext) != n + 2:
            break
        x = grid[ext]
    return c


def fit(n: int = 3):
    c32 = remez(n).astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001)
    err = np.max(np.abs(np.polyval(c32[::-1].astype(np.float64), grid) / 2.0 ** grid - 1))
    return c32, float(err)


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"kExp2C{i} = {float(v)!r}f")
    print(f"max relative error on [-0.5, 0.5]: {e:.3e}")
