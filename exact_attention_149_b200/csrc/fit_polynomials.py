"""Derive the polynomial the kernels evaluate on the FMA pipe.

A minimax fit (Remez exchange algorithm, minimal maximum *relative* error)
written for this library: tanh(y) = y * Q(y^2) for |y| <= 0.5, Q of degree 4
on t = y^2 in [0, 0.25], of degree 2 for |y| <= 0.25 and of degree 1 for
|y| <= 0.125, used for softcap when every |y| of a warp's rows is small. The same routine also gives the degree-3 fit of 2^f on [-0.5, 0.5]
(relative error 7.5e-5) that the forward kernel evaluates for a quarter of
its exponentials (ex2_poly2), moving that share of the work from the
special-function unit, which bounds the softmax, to the FMA pipe.

    python exact_attention_149_b200/csrc/fit_polynomials.py

prints the coefficients (copied into ptx.cuh) and the float32 evaluation
error against numpy's float64 functions.
"""

import numpy as np


def remez(f, n, a, b, iters=60):
    """Minimax polynomial of degree n for f on [a, b] (relative error)."""
    m = n + 2
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * np.arange(m) / (m - 1))
    grid = np.linspace(a, b, 400001)
    c = None
    for _ in range(iters):
        mat = np.zeros((m, m))
        for i in range(m):
            mat[i, :n + 1] = x[i] ** np.arange(n + 1)
            mat[i, n + 1] = (-1) ** i * f(np.array([x[i]]))[0]
        c = np.linalg.solve(mat, f(x))[:n + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        runs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < m:
            break
        if len(ext) > m:
            ext = sorted(sorted(ext, key=lambda i: -abs(err[i]))[:m])
        x = grid[ext]
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.max(np.abs(err)))


def horner32(c, x):
    c32 = c.astype(np.float32)
    q = np.float32(c32[-1]) * np.ones_like(x)
    for k in range(len(c32) - 2, -1, -1):
        q = (q * x + c32[k]).astype(np.float32)
    return q


def tanh_ratio(t):
    t = np.asarray(t, dtype=np.float64)
    y = np.sqrt(t)
    out = np.ones_like(t)
    nz = y > 1e-8
    out[nz] = np.tanh(y[nz]) / y[nz]
    return out


if __name__ == "__main__":
    c, e = remez(tanh_ratio, 4, 0.0, 0.25)
    print("tanh: Q(t), t = y^2 in [0, 0.25]; max relative error (float64):", e)
    for k, v in enumerate(c):
        print(f"  q{k} = {v:.9e}f")
    y = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    th = (y * horner32(c, (y * y).astype(np.float32))).astype(np.float32)
    print("  float32 max abs error:", float(np.max(np.abs(th - np.tanh(y.astype(np.float64))))))

    c, e = remez(tanh_ratio, 2, 0.0, 0.0625)
    print("tanh: Q(t), t = y^2 in [0, 1/16] (|y| <= 1/4); max relative error (float64):", e)
    for k, v in enumerate(c):
        print(f"  q{k} = {v:.9e}f")
    y = np.linspace(-0.25, 0.25, 400001).astype(np.float32)
    th = (y * horner32(c, (y * y).astype(np.float32))).astype(np.float32)
    print("  float32 max abs error:", float(np.max(np.abs(th - np.tanh(y.astype(np.float64))))))

    c, e = remez(tanh_ratio, 1, 0.0, 0.015625)
    print("tanh: Q(t), t = y^2 in [0, 1/64] (|y| <= 1/8); max relative error (float64):", e)
    for k, v in enumerate(c):
        print(f"  q{k} = {v:.9e}f")
    y = np.linspace(-0.125, 0.125, 400001).astype(np.float32)
    th = (y * horner32(c, (y * y).astype(np.float32))).astype(np.float32)
    print("  float32 max abs error:", float(np.max(np.abs(th - np.tanh(y.astype(np.float64))))))

    c, e = remez(np.exp2, 3, -0.5, 0.5)
    print("exp2: E(f), f in [-0.5, 0.5]; max relative error (float64):", e)
    for k, v in enumerate(c):
        print(f"  e{k} = {v:.9e}f")
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    print("  float32 max rel error:", float(np.max(np.abs(horner32(c, f) - ref) / ref)))
