"""Reproduces the degree-3 exp2 polynomial used by the attention kernel's softmax.

2^x = 2^n * 2^f with n = round(x) and f in [-0.5, 0.5]; 2^f is approximated by the degree-3
polynomial that minimises the maximum RELATIVE error on [-0.5, 0.5] (Remez exchange algorithm:
solve for coefficients that make the weighted error equioscillate on deg+2 reference points, move
the references to the error extrema, repeat). Coefficients are rounded to float32; the script
prints them and the maximum relative error of the float32 Horner evaluation.

    python block_sparse_long_causal_b200/exp2_fit.py
"""
import numpy as np


def remez_exp2(deg=3, a=-0.5, b=0.5, iters=40, grid=400001):
    m = deg + 2
    x = np.array([(a + b) / 2 - (b - a) / 2 * np.cos(np.pi * k / (m - 1)) for k in range(m)])
    g = np.linspace(a, b, grid)
    c = None
    for _ in range(iters):
        A = np.zeros((m, m))
        rhs = 2.0 ** x
        A[:, : deg + 1] = x[:, None] ** np.arange(deg + 1)
        A[:, deg + 1] = (-1.0) ** np.arange(m) * rhs
        c = np.linalg.solve(A, rhs)[: deg + 1]
        err = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        ext = [0] + [i for i in range(1, grid - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) < 0] + [grid - 1]
        if len(ext) != m:
            break
        x = g[ext]
    c32 = c.astype(np.float32)
    gf = g.astype(np.float32)
    acc = np.full_like(gf, c32[deg])
    for k in range(deg - 1, -1, -1):
        acc = (acc * gf + c32[k]).astype(np.float32)
    rel = np.abs(acc.astype(np.float64) / 2.0 ** gf.astype(np.float64) - 1.0).max()
    return c32, float(rel)


if __name__ == "__main__":
    coef, rel = remez_exp2()
    for i, v in enumerate(coef):
        print(f"c{i} = {float(v)!r}")
    print(f"max relative error (float32 Horner) = {rel:.3e}")
