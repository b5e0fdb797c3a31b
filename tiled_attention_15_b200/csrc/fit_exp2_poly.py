"""Fit of the polynomial behind the kernels' FMA-pipe exp2 (run: python fit_exp2_poly.py).

2^x is computed as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2];
2^f is approximated by the polynomial of degree 3 that minimises the maximum
relative error on that interval, found here with the Remez exchange
algorithm.  The printed float32 coefficients are the ones in sm100_ptx.cuh
(kExp2C0..kExp2C3); the float32 Horner evaluation error (~7.5e-5 relative)
is the bound the tests check.
"""
import numpy as np
def remez(n, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative)
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, :n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * f(xi)
        c = np.linalg.solve(A, f(x))
        coef, E = c[:n + 1], c[n + 1]
        g = np.linspace(a, b, 200001)
        err = (np.polyval(coef[::-1], g) - f(g)) / f(g)
        # new reference: extrema of err between sign changes
        idx = [0]
        s = np.sign(err)
        ext = []
        start = 0
        for i in range(1, len(g)):
            if s[i] != s[i - 1]:
                seg = slice(start, i)
                j = start + np.argmax(np.abs(err[seg])); ext.append(j); start = i
        j = start + np.argmax(np.abs(err[start:])); ext.append(j)
        if len(ext) != n + 2:
            break
        x = g[ext]
    return coef, np.abs(err).max()
for n in (3,):
    c, e = remez(n)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    # evaluate in float32 Horner like the kernel
    p = np.float32(c32[n])
    for k in range(n - 1, -1, -1):
        p = (p * g + c32[k]).astype(np.float32)
    e32 = np.abs((p.astype(np.float64) - np.exp2(g.astype(np.float64))) / np.exp2(g.astype(np.float64))).max()
    print(n, "rel err (exact coef)", e, "float32 Horner", e32, "coefs", [float(v) for v in c32])
