"""Fit the cubic used by exp2_poly2 (sm100_ptx.cuh) for 2^f on [-1/2, 1/2].

Remez exchange on the relative error p(f)/2^f - 1: solve for the cubic whose
error equioscillates at five points, move the points to the extrema of the
new error curve, repeat.  Run it to reproduce the constants:

    python tiled_exact_attention_fa_b200/csrc/fit_exp2_poly.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def fit(iterations: int = 40, grid: int = 200001):
    f = np.linspace(LO, HI, grid)
    target = np.exp2(f)
    n = DEGREE + 2
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.linspace(np.pi, 0, n))
    coeffs = None
    for _ in range(iterations):
        A = np.zeros((n, n))
        b = np.exp2(nodes)
        for i, x in enumerate(nodes):
            A[i, :DEGREE + 1] = [x ** k for k in range(DEGREE + 1)]
            A[i, DEGREE + 1] = -((-1) ** i) * np.exp2(x)
        coeffs = np.linalg.solve(A, b)[:DEGREE + 1]
        err = np.polyval(coeffs[::-1], f) / target - 1.0
        # one extremum per run of constant sign
        sign = np.sign(err)
        ext, i = [], 0
        while i < grid:
            j = i
            while j < grid and sign[j] == sign[i]:
                j += 1
            ext.append(i + int(np.argmax(np.abs(err[i:j]))))
            i = j
        if len(ext) != n:
            ext = sorted(sorted(ext, key=lambda k: -abs(err[k]))[:n])
        nodes = f[ext]
    err = np.polyval(coeffs[::-1], f) / target - 1.0
    return coeffs, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = fit()
    c32 = np.asarray(c, dtype=np.float32)
    for k, v in enumerate(c32):
        print(f"kExp2C{k} = {float(v).hex()}  ({float(v):.9g})")
    print(f"max relative error {e:.3e} (2^{np.log2(e):.2f})")
