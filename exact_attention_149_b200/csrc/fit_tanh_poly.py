"""Derive the polynomial the kernels use for tanh on small arguments.

tanh(y) = y * Q(y^2) for |y| <= 0.5, with Q a degree-4 polynomial chosen by
the Remez exchange algorithm to minimise the maximum *relative* error of
tanh(sqrt t)/sqrt t on t in [0, 0.25]. The kernels evaluate Q with fused
multiply-adds (packed two at a time) instead of the two special-function
operations of the exp-based identity, and fall back to that identity for any
row whose largest |y| exceeds 0.5.

    python exact_attention_149_b200/csrc/fit_tanh_poly.py

prints the coefficients (copied into ptx.cuh) and the float32 error over
[-0.5, 0.5] against numpy's float64 tanh.
"""

import numpy as np

T = 0.25    # t = y^2 range
DEG = 4


def f(t):
    t = np.asarray(t, dtype=np.float64)
    y = np.sqrt(t)
    out = np.ones_like(t)
    nz = y > 1e-8
    out[nz] = np.tanh(y[nz]) / y[nz]
    return out


def remez(n, iters=60):
    m = n + 2
    x = (T / 2) * (1 - np.cos(np.pi * np.arange(m) / (m - 1)))
    grid = np.linspace(0, T, 400001)
    for _ in range(iters):
        a = np.zeros((m, m))
        for i in range(m):
            a[i, :n + 1] = x[i] ** np.arange(n + 1)
            a[i, n + 1] = (-1) ** i * f(x[i:i + 1])[0]
        sol = np.linalg.solve(a, f(x))
        c = sol[:n + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        runs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < m:
            break
        if len(ext) > m:
            ext = sorted(sorted(ext, key=lambda i: -abs(err[i]))[:m])
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez(DEG)
    print("max relative error (float64):", e)
    for k, v in enumerate(c):
        print(f"c{k} = {v:.9e}f")
    c32 = c.astype(np.float32)
    y = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    t = (y * y).astype(np.float32)
    q = np.float32(c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        q = (q * t + c32[k]).astype(np.float32)
    th = (y * q).astype(np.float32)
    ref = np.tanh(y.astype(np.float64))
    print("float32 max abs error:", float(np.max(np.abs(th - ref))))
