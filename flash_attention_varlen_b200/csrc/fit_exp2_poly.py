"""Fits the polynomial the bf16 kernel uses to evaluate part of its exp2s on the FMA pipe.

Method (Cody-Waite range reduction + minimax polynomial):
  x = n + f with n = round(x) and f in [-1/2, 1/2]   (round via the 1.5*2^23 shift)
  2^x = 2^n * 2^f, 2^n by adding n to the float exponent field,
  2^f ~ p(f), p of degree `deg` minimising the maximum RELATIVE error on
  [-1/2, 1/2], found with the Remez exchange algorithm (float64/longdouble).

    python -m flash_attention_varlen_b200.csrc.fit_exp2_poly [deg]

prints the coefficients (low order first) as C float literals and the achieved
maximum relative error, before and after rounding the coefficients to float32.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 60):
    a, b = -0.5, 0.5
    n = deg + 2
    # initial reference: Chebyshev extrema
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve  sum_k c_k x_i^k - (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((n, n))
        for k in range(deg + 1):
            A[:, k] = x ** k
        A[:, deg + 1] = -((-1.0) ** np.arange(n)) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extrema of err on each sign-alternating run
        sign = np.sign(err)
        idx = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sign[i] != sign[start]:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        if len(idx) < n:
            break
        # keep the n largest consecutive alternation points
        idx = np.array(idx)
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx = idx[1:]
            else:
                idx = idx[:-1]
        x_new = grid[idx]
        if np.allclose(x_new, x, atol=1e-12):
            break
        x = x_new
    return c, float(np.max(np.abs(err)))


def max_rel_err_f32(coef32) -> float:
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for ck in coef32[-2::-1]:
        p = (p * f + ck).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    c32 = c.astype(np.float32)
    print(f"degree {deg}: max relative error {e:.3e} (float64 coefficients), "
          f"{max_rel_err_f32(c32):.3e} (float32 coefficients, float32 Horner)")
    for k, ck in enumerate(c32):
        print(f"  c{k} = {float(ck).hex()}  // {float(ck):.9e}")


if __name__ == "__main__":
    main()
