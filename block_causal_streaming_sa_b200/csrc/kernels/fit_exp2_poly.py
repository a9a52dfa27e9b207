"""Fit of the polynomial behind ptx::exp2_poly (kernels/ptx.cuh).

2^f on [-1/2, 1/2] by a degree-3 polynomial, minimax in relative error, found
with the Remez exchange algorithm (equioscillation of the relative error at
deg + 2 reference points, reference moved to the error's extrema each pass).
Prints the coefficients (float32) and the max relative error of the float32
Horner evaluation; the kernel's constants are these values.

    python block_causal_streaming_sa_b200/csrc/kernels/fit_exp2_poly.py
"""

import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k / (n - 1))[::-1]
    t = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], t) - np.exp2(t)) / np.exp2(t)
        ext, start, sgn = [], 0, np.sign(err)
        for j in range(1, len(t)):
            if sgn[j] != sgn[j - 1]:
                seg = np.arange(start, j)
                ext.append(seg[np.argmax(np.abs(err[seg]))])
                start = j
        seg = np.arange(start, len(t))
        ext.append(seg[np.argmax(np.abs(err[seg]))])
        ext = np.array(ext)
        if len(ext) >= n:
            best = max(range(len(ext) - n + 1), key=lambda s: np.min(np.abs(err[ext[s:s + n]])))
            x = t[ext[best:best + n]]
    return c


def horner32(c, t):
    c32 = c.astype(np.float32)
    p = np.full_like(t, c32[-1])
    for cc in c32[-2::-1]:
        p = (p * t + cc).astype(np.float32)
    return p


if __name__ == "__main__":
    c = remez(3)
    t = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    ref = np.exp2(t.astype(np.float64))
    err = np.max(np.abs(horner32(c, t) - ref) / ref)
    print("coefficients c0..c3:", [float(np.float32(v)) for v in c])
    print(f"max relative error (float32 Horner): {err:.3e}")
