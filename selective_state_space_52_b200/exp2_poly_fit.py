"""Coefficients of the FMA-pipe exp2 in csrc/device_math.cuh (exp2_fma).

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody and
Waite's argument reduction, exact here: n is an integer and f is formed by one
float32 subtraction of a representable integer), and 2^f approximated by the
degree-6 polynomial with constant term 1 (so that 2^0 is exactly 1: a masked
token's decay) that minimises the largest relative error on [-1/2, 1/2]
(Remez's exchange algorithm, relative weight 1 / 2^f).  The fit runs in
float64; the coefficients are then rounded to float32, and the float32 Horner
evaluation of the rounded polynomial is what the tests measure.

    python -m selective_state_space_52_b200.exp2_poly_fit
prints the coefficients (c0 .. c6) and the float32 evaluation's worst
relative error.
"""
from __future__ import annotations

import numpy as np

DEGREE = 6
LO, HI = -0.5, 0.5


def _solve(nodes: np.ndarray) -> tuple[np.ndarray, float]:
    """Polynomial c (c0 = 1) and level E with (p(x_i) - 2^x_i) / 2^x_i = (-1)^i E."""
    n = DEGREE + 1
    A = np.zeros((n, n))
    rhs = np.exp2(nodes) - 1.0
    for i, x in enumerate(nodes):
        A[i, :DEGREE] = x ** np.arange(1, DEGREE + 1)
        A[i, DEGREE] = -((-1) ** i) * np.exp2(x)
    sol = np.linalg.solve(A, rhs)
    return np.concatenate([[1.0], sol[:DEGREE]]), float(sol[DEGREE])


def remez(iterations: int = 30, grid: int = 200001) -> np.ndarray:
    """Remez exchange for the relative-error minimax polynomial of 2^x."""
    k = np.arange(DEGREE + 1)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (DEGREE - k) / DEGREE)
    nodes = nodes + 1e-3 * (nodes == 0)          # the error is zero at 0 itself
    xs = np.linspace(LO, HI, grid)
    c = None
    for _ in range(iterations):
        c, _ = _solve(nodes)
        err = np.polynomial.polynomial.polyval(xs, c) / np.exp2(xs) - 1.0
        # one extremum per sign run of the error (the forced zero at 0 does not
        # alternate: runs are split where the sign changes away from it)
        sign = np.sign(err)
        sign[sign == 0] = 1
        cuts = np.nonzero(np.diff(sign) != 0)[0] + 1
        runs = np.split(np.arange(grid), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < DEGREE + 1:
            break
        # keep the DEGREE + 1 alternating extrema of largest magnitude
        while len(ext) > DEGREE + 1:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext.pop(drop)
        new = xs[np.array(ext)]
        if np.allclose(new, nodes, atol=1e-12):
            nodes = new
            break
        nodes = new
    return c


def horner_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """The float32 Horner evaluation the kernel performs (fused multiply-add
    emulated in float64, then rounded to float32, which is exact for one
    product and one sum of float32 values)."""
    f = f.astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return p


def coefficients() -> np.ndarray:
    return remez().astype(np.float32)


if __name__ == "__main__":
    c32 = coefficients()
    f = np.linspace(LO, HI, 1000001).astype(np.float32)
    rel = np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v):.9e}f  ({float(v).hex()})")
    print(f"worst relative error of the float32 evaluation on [-1/2, 1/2]: {rel.max():.3e} "
          f"({rel.max() / 2.0 ** -24:.2f} x 2^-24)")
