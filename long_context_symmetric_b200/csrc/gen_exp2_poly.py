"""Coefficients of the FMA-pipe 2^x used by the attention softmax (tc_ptx.cuh).

2^x = 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2]: for base 2 the
Cody-Waite range reduction is exact in binary floating point, since n is an
integer and f is formed without rounding. 2^f is a degree-5 polynomial with
minimax RELATIVE error on [-1/2, 1/2], found by the Remez exchange algorithm
(solve for the polynomial that equioscillates on n+2 reference points, move the
points to the extrema of the error, repeat) in 50-digit arithmetic, then rounded
to fp32. Run: python gen_exp2_poly.py  (needs mpmath; prints the coefficients and
the error of the fp32 Horner evaluation on a dense grid).
"""

import mpmath as mp
import numpy as np

mp.mp.dps = 50


def remez_exp2(deg: int, a=-0.5, b=0.5, iters=40, grid=4000):
    m = deg + 2
    xs = [mp.mpf(a + b) / 2 + mp.mpf(b - a) / 2 * mp.cos(mp.pi * (m - 1 - i) / (m - 1)) for i in range(m)]
    for _ in range(iters):
        A = mp.matrix(m, m)
        rhs = mp.matrix(m, 1)
        for i, x in enumerate(xs):
            for k in range(deg + 1):
                A[i, k] = x ** k
            A[i, deg + 1] = (-1) ** i * mp.power(2, x)      # p(x) - 2^x = (-1)^i E 2^x
            rhs[i] = mp.power(2, x)
        sol = mp.lu_solve(A, rhs)
        c = [sol[k] for k in range(deg + 1)]
        err = lambda x: sum(c[k] * x ** k for k in range(deg + 1)) / mp.power(2, x) - 1
        pts = [mp.mpf(a) + (mp.mpf(b) - a) * j / grid for j in range(grid + 1)]
        vals = [err(x) for x in pts]
        ext = [pts[0]] + [pts[j] for j in range(1, grid)
                          if (vals[j] - vals[j - 1]) * (vals[j + 1] - vals[j]) <= 0] + [pts[-1]]
        if len(ext) == m:
            xs = ext
    return c, max(abs(v) for v in vals)


def fp32_horner_error(c32):
    x = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    acc = np.full_like(x, c32[-1])
    for ck in reversed(c32[:-1]):
        acc = (acc.astype(np.float64) * x.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return float(np.max(np.abs(acc.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)))


if __name__ == "__main__":
    c, e = remez_exp2(5)
    c32 = [np.float32(float(v)) for v in c]
    print(f"minimax relative error 2^{float(mp.log(e, 2)):.2f}; fp32 Horner 2^{np.log2(fp32_horner_error(c32)):.2f}")
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v)!r}f")
