"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2].

The attention kernel computes part of its softmax exponentials on the FMA
pipe instead of the MUFU unit: 2^x = 2^n * 2^f with n = round(x) (Cody-Waite
range reduction, here with a single exact step since the base is 2) and
2^f from this cubic.  The cubic is the minimax approximation of 2^f for
RELATIVE error on [-1/2, 1/2], found by the Remez exchange algorithm below
(fp64, numpy); its maximum relative error is about 7.5e-5, far below the
bf16 rounding (2^-9 = 2e-3) the softmax weights then take.

Run `python -m rank_latent_attention_mixer_b200.exp2_poly` to print the
coefficients as fp32 literals; tests/test_exp2_poly.py checks that the
constants in csrc/kernels_tc.cuh are these.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(nodes: np.ndarray, degree: int):
    """Coefficients c and level E with (p(x_i) - 2^x_i) / 2^x_i = (-1)^i E at the nodes."""
    n = degree + 2
    A = np.zeros((n, n))
    b = np.exp2(nodes)
    for i, x in enumerate(nodes):
        A[i, : degree + 1] = x ** np.arange(degree + 1)
        A[i, degree + 1] = (-1) ** i * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[: degree + 1], sol[degree + 1]


def remez(degree: int = DEGREE, iters: int = 50):
    """Minimax (relative error) polynomial for 2^f on [LO, HI]."""
    k = np.arange(degree + 2)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (degree + 1))  # Chebyshev extrema
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        c, _ = _solve(nodes, degree)
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new nodes: the extremum of each sign-alternating run of the error
        sign = np.sign(err)
        breaks = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(grid.size), breaks)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < degree + 2:
            break
        ext = sorted(ext, key=lambda i: -abs(err[i]))[: degree + 2]
        new = np.sort(grid[ext])
        if np.allclose(new, nodes, atol=1e-12):
            break
        nodes = new
    c, _ = _solve(nodes, degree)
    err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
    return c, float(np.abs(err).max())


def coefficients_f32():
    c, _ = remez()
    return [float(np.float32(v)) for v in c]


def max_rel_error_f32() -> float:
    """Relative error of the fp32-rounded cubic, evaluated in fp64 (Horner)."""
    c = np.array(coefficients_f32())
    f = np.linspace(LO, HI, 200001)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    return float(np.abs((p - np.exp2(f)) / np.exp2(f)).max())


if __name__ == "__main__":
    c, e = remez()
    print("fp64 coefficients:", ", ".join(repr(float(v)) for v in c), f"max rel err {e:.3e}")
    print("fp32 literals:", ", ".join(f"{v!r}f" for v in coefficients_f32()),
          f"max rel err {max_rel_error_f32():.3e}")
