"""Fits the polynomial the kernel uses to evaluate part of its 2^x on the FMA pipe.

Method (classical range reduction plus a minimax polynomial):
  x = n + f with n = round(x) and f in [-1/2, 1/2];  2^x = 2^n * 2^f;
  2^f ~= c0 + c1 f + c2 f^2 + c3 f^3, with the coefficients chosen by the Remez
  exchange algorithm to minimise the maximum RELATIVE error on [-1/2, 1/2].
The 2^n factor is applied by adding n to the float's exponent field.

Run it to print the float32 coefficients and the worst relative error of a
float32 Horner evaluation over a dense grid:

    python exact_tiled_attention_44_b200/csrc/fit_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def remez_rel(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    """Minimax (relative error) polynomial for 2^f on [lo, hi]."""
    n = degree + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of err in each sign-alternating segment
        sign = np.sign(err)
        idx = np.where(np.diff(sign) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [grid.size]])
        ext = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            seg = np.abs(err[a:b])
            ext.append(a + int(np.argmax(seg)))
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext.pop(0)
            else:
                ext.pop()
        x = grid[np.array(ext)]
    return coef


def f32_exp2(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """float32 model of the kernel's evaluation: round-to-nearest adds, and one
    rounding per fused multiply-add (product and sum formed in float64)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)          # 1.5 * 2^23: adding it rounds x to an integer
    t = (x + magic).astype(np.float32)
    u = (t - magic).astype(np.float32)
    f = (x - u).astype(np.float32)
    p = np.full_like(f, np.float32(c[-1]))
    for ci in c[-2::-1]:
        p = (p.astype(np.float64) * f + np.float64(np.float32(ci))).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez_rel(deg).astype(np.float32)
    xs = np.linspace(-120.0, 8.0, 2_000_001).astype(np.float32)
    y = f32_exp2(xs, c).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    print("coefficients (float32):", ", ".join(f"{v:.9e}f" for v in c))
    print(f"max relative error on [-120, 8]: {rel.max():.3e} (bf16 half-ulp is {2**-9:.3e})")


if __name__ == "__main__":
    main()
