"""Fit the polynomial the attention kernel uses for part of its 2^f evaluations.

Method: minimax (Remez exchange) fit of p(f) ~= 2^f on f in [-1/2, 1/2] with
RELATIVE error weight, degree 3, all four coefficients free. The kernel writes 2^x = p(x - n) * 2^n with n = round(x) and builds
2^n from its exponent bits, so only the reduced argument needs the
polynomial. Run this file to print the coefficients that csrc/attn_sm100.cuh
embeds (in single precision) and the maximum relative error of the
single-precision Horner evaluation.
"""
import numpy as np


def remez_rel(deg=3, lo=-0.5, hi=0.5, iters=30):
    # p(f) = c0 + c1 f + ... + c_deg f^deg ; minimise max |p/2^f - 1|
    n = deg + 1  # unknowns c0..c_deg, plus the levelled error E
    pts = np.cos(np.linspace(np.pi, 0, n + 1)) * (hi - lo) / 2 + (hi + lo) / 2
    grid = np.linspace(lo, hi, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n + 1, n + 1))
        b = np.zeros(n + 1)
        for i, x in enumerate(pts):
            t = 2.0 ** x
            for k in range(0, deg + 1):
                A[i, k] = x ** k / t
            A[i, n] = (-1) ** i
            b[i] = 1.0
        sol = np.linalg.solve(A, b)
        c = sol[:n]
        err = sum(c[k] * grid ** k for k in range(0, deg + 1)) / 2.0 ** grid - 1
        # new reference points: extrema of the error curve, alternating in sign
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        cand = sorted(idx, key=lambda j: -abs(err[j]))
        chosen = sorted(cand[:n + 1])
        pts = grid[chosen]
    return c, float(np.max(np.abs(err)))


def horner_f32(coef, f):
    f = np.float32(f)
    r = np.float32(coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        r = np.float32(np.float32(r * f) + np.float32(coef[k]))
    return r


if __name__ == "__main__":
    coef, e = remez_rel()
    c32 = [np.float32(x) for x in coef]
    fs = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    vals = np.array([horner_f32(c32, f) for f in fs[::50]])
    rel = np.max(np.abs(vals.astype(np.float64) / 2.0 ** fs[::50].astype(np.float64) - 1))
    print("coefficients c0..c3 (fp32):", ", ".join(f"{float(x):.9e}f" for x in c32))
    print(f"minimax relative error (exact arithmetic): {e:.3e}")
    print(f"relative error of the fp32 Horner evaluation (sampled): {rel:.3e}")
