"""Fits the polynomial the attention kernels use for part of their 2^x
evaluations on the FMA pipe (the rest run on the MUFU ex2 unit).

Method: Cody-Waite style range reduction x = n + f with n = round(x),
f in [-1/2, 1/2], 2^x = 2^n * P(f); P is the degree-3 minimax polynomial of
2^f on [-1/2, 1/2] in relative error, found here by the Remez exchange
algorithm and rounded to fp32.  Run it to reprint the coefficients and their
error (degree 3: max relative error 7.5e-5, far below bf16's 2^-8 step).
"""
import numpy as np
def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (b - a) / 2 + (a + b) / 2
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E * 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:deg + 1], sol[deg + 1]
        g = np.linspace(a, b, 20001)
        err = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        # new extrema: endpoints + interior sign-change extrema
        idx = [0]
        for i in range(1, len(g) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) < 0:
                idx.append(i)
        idx.append(len(g) - 1)
        if len(idx) != n:
            break
        x = g[idx]
    return c, np.abs(err).max()
for d in (3,):
    c, e = remez(d)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(g)
    for ci in c32[::-1]:
        p = p * g + ci           # Horner in fp32 (fma-free approx)
    rel = np.abs(p.astype(np.float64) / 2.0 ** g.astype(np.float64) - 1).max()
    print(d, [float(v) for v in c32], 'minimax rel err', e, 'fp32 eval', rel)
