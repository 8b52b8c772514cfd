"""Derives the polynomial used by exp2_poly() in sm100_ptx.cuh.

Method: Cody-Waite style range reduction (W. J. Cody and W. Waite, "Software
Manual for the Elementary Functions", 1980): 2^x = 2^n * 2^f with n = round(x)
and f = x - n in [-1/2, 1/2]; 2^n is built as a float from its exponent field and
applied by one multiplication.  2^f is approximated by the cubic p(f) = c0 + c1 f + c2 f^2 + c3 f^3
whose maximum *relative* error on [-1/2, 1/2] is minimised with the Remez
exchange algorithm (E. Ya. Remez, 1934) on the weighted Haar system
{1, f, f^2, f^3} * 2^-f.  (Pinning c0 = 1 would make every basis function but
one vanish at f = 0, which is not a Haar system, so c0 is left free.)

    python exact_attention_107_b200/csrc/gen_exp2_poly.py

prints the coefficients (as float32 hex) and the maximum relative error of the
float32 evaluation over a dense grid.  The kernels only need the printed values;
this script documents where they come from and is not part of the build.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int, iters: int = 50):
    """Coefficients c0..c_degree minimising max |p(f) / 2^f - 1| on [LO, HI]."""
    m = degree + 1                      # unknown coefficients; plus the levelled error E
    k = np.arange(m + 1)
    ref = (LO + HI) / 2 - (HI - LO) / 2 * np.cos(np.pi * k / m)     # Chebyshev extrema
    grid = np.linspace(LO, HI, 400001)
    basis = lambda f: np.stack([f ** j for j in range(m)], axis=-1)
    coef = None
    for _ in range(iters):
        # p(f_i) 2^-f_i - 1 = (-1)^i E at the m+1 reference points
        A = np.concatenate([basis(ref) * (2.0 ** -ref)[:, None], -((-1.0) ** k)[:, None]], axis=1)
        sol = np.linalg.solve(A, np.ones(m + 1))
        coef = sol[:m]
        err = basis(grid) @ coef * 2.0 ** -grid - 1.0
        # exchange: one extremum of |err| per run of constant sign, keep m+1 of them
        runs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        while len(ext) > m + 1:
            ext.pop(0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else -1)
        if len(ext) < m + 1:
            break
        new_ref = grid[ext]
        if np.allclose(new_ref, ref):
            break
        ref = new_ref
    return coef


def eval_f32(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernels' steps in float32: NaN-keeping clamp, round-to-integer by adding
    1.5*2^23 + 127 (the sum's low 9 mantissa bits are then n + 127), f = x - n, Horner
    polynomial, times 2^n made from those bits as an exponent field."""
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))      # numpy's maximum keeps NaN
    magic = np.float32(12583039.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = c.astype(np.float32)
    p = c[3] * f + c[2]
    p = p.astype(np.float32) * f + c[1]
    p = p.astype(np.float32) * f + c[0]
    scale = (t.view(np.int32) << 23).astype(np.int32).view(np.float32)
    with np.errstate(invalid="ignore", over="ignore"):
        return (p.astype(np.float32) * scale).astype(np.float32)


if __name__ == "__main__":
    c = remez_relative(DEGREE)
    c32 = c.astype(np.float32)
    print("coefficients c0..c3 (float32):", [float(v) for v in c32], [v.tobytes()[::-1].hex() for v in c32])
    xs = np.linspace(-125.0, 10.0, 4_000_001)
    got = eval_f32(xs, c32).astype(np.float64)
    rel = np.abs(got / np.exp2(xs) - 1.0)
    print(f"max relative error over [-125, 10]: {rel.max():.3e}")
