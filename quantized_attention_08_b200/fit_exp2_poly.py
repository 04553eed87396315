"""Fit the polynomial the attention kernel uses for 2^r on [-1/2, 1/2].

    python -m quantized_attention_08_b200.fit_exp2_poly [degree]

The kernel evaluates part of each row's exponentials on the FMA pipe:
x = n + r with n = rint(x), r in [-1/2, 1/2] (exact in fp32), 2^r by a
polynomial, 2^n added into the exponent field.  This script fits that
polynomial by a Remez exchange that equalises the RELATIVE error
(p(r) - 2^r) / 2^r over the interval, prints the coefficients as fp32
literals for csrc/attn_sm100.cu (kExpC0..kExpC5) and reports the maximum
relative error of the fp32 Horner evaluation.  It is a development tool: the
library does not run it.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_relative(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    """Coefficients c[0..deg] (ascending) of the minimax-relative-error
    polynomial for 2^r on [lo, hi], and the levelled error."""
    n = deg + 2
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 400001)
    f = np.exp2
    c = None
    for _ in range(iters):
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            a[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(a, f(x))
        c = sol[:deg + 1]
        err = (np.polynomial.polynomial.polyval(grid, c) - f(grid)) / f(grid)
        # one extremum per run of equal sign
        edges = np.nonzero(np.diff(np.sign(err)) != 0)[0] + 1
        runs = np.split(np.arange(len(grid)), edges)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.abs(err).max())


def horner_fp32(c, r):
    """Horner evaluation with one rounding to fp32 per fused multiply-add
    (product exact in fp64, sum rounded to fp64 then to fp32)."""
    c32 = [np.float32(v) for v in c]
    r = np.asarray(r, np.float32)
    p = np.full(r.shape, c32[-1], np.float32)
    for v in c32[-2::-1]:
        p = (p.astype(np.float64) * r.astype(np.float64) + np.float64(v)).astype(np.float32)
    return p


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c, lev = remez_relative(deg)
    r = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    p = horner_fp32(c, r)
    exact = np.exp2(r.astype(np.float64))
    e32 = float(np.abs((p.astype(np.float64) - exact) / exact).max())
    print(f"// degree {deg}: levelled relative error {lev:.3e} (2^{np.log2(lev):.2f}), "
          f"fp32 Horner {e32:.3e} (2^{np.log2(e32):.2f})")
    for i, v in enumerate(c):
        print(f"constexpr float kExpC{i} = {float(np.float32(v)):.17e}f;")


if __name__ == "__main__":
    main()
