"""Coefficients of the cubic that exp2_fma2 (seg_attn.cu) uses for 2^f, f in [-1/2, 1/2].

The softmax moves part of its exponentials from the MUFU unit to the FMA pipe:
x = n + f with n = rint(x), 2^x = 2^n * 2^f, and 2^f by a polynomial. This
script finds the cubic c0 + c1 f + c2 f^2 + c3 f^3 that minimises the maximum
RELATIVE error max |p(f) / 2^f - 1| over [-1/2, 1/2], as a linear program on a
dense grid (variables c0..c3 and the bound E; |p(f_i) - 2^f_i| <= E 2^f_i),
then rounds the coefficients to fp32 and reports the error of the fp32 Horner
evaluation. Run it to reprint the constants:

    python tests/tools/exp2_poly_fit.py
"""

from __future__ import annotations

import numpy as np


def fit(degree: int = 3, points: int = 4001) -> tuple[np.ndarray, float]:
    """Minimax-relative-error coefficients (fp32, lowest order first) and their fp64 LP bound."""
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    cost = np.zeros(degree + 2)
    cost[-1] = 1.0
    r = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)], method="highs")
    if not r.success:
        raise RuntimeError(r.message)
    return r.x[:-1].astype(np.float32), float(r.x[-1])


def horner_f32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """fp32 Horner evaluation with one rounding per fused multiply-add (as the kernel's FFMA2)."""
    f = f.astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c[k])).astype(np.float32)
    return p


if __name__ == "__main__":
    c, bound = fit()
    grid = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(horner_f32(c, grid).astype(np.float64) / np.exp2(grid.astype(np.float32).astype(np.float64)) - 1)
    for k, v in enumerate(c):
        print(f"constexpr float kExp2C{k} = {float(v)!r}f;")
    print(f"// max relative error: LP bound {bound:.3e}, fp32 evaluation {err.max():.3e}")
