"""Derives the cubic of exp2_poly2 (the FMA-pipe 2^x of the tensor-core score passes).

2^x for x <= 0 is split Cody-Waite style as 2^j 2^f with j = rint(x) and f = x - j in
[-1/2, 1/2]; 2^f comes from a cubic p(f) = ((c3 f + c2) f + c1) f + c0. The coefficients are
the minimax approximation of 2^f on [-1/2, 1/2] in *relative* error, max |p(f) / 2^f - 1|,
found here by the Remez exchange algorithm: on a reference of five points solve
p(x_i) - 2^x_i = (-1)^i E 2^x_i for the four coefficients and the levelled error E, move the
reference to the extrema of the error curve, repeat until the extrema are level.

Run as a script it prints the coefficients (float32) and the error bound; the tests call fit().
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(ref: np.ndarray):
    n = DEGREE + 1
    A = np.zeros((n + 1, n + 1))
    b = np.exp2(ref)
    for i, x in enumerate(ref):
        A[i, :n] = x ** np.arange(n)
        A[i, n] = (-1) ** i * np.exp2(x)
    sol = np.linalg.solve(A, b)
    return sol[:n], sol[n]


def _rel_err(c: np.ndarray, x: np.ndarray) -> np.ndarray:
    return np.polyval(c[::-1], x) / np.exp2(x) - 1.0


def fit(iters: int = 50, grid: int = 200001):
    """Remez exchange for the relative-error minimax cubic; returns (coefficients c0..c3 as
    float64, levelled error |E|)."""
    n = DEGREE + 2
    # Chebyshev extrema as the first reference
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    xs = np.linspace(LO, HI, grid)
    c, E = _solve(ref)
    for _ in range(iters):
        c, E = _solve(ref)
        e = _rel_err(c, xs)
        # one extremum per sign run of the error curve (the ends included)
        sign = np.sign(e)
        cuts = np.nonzero(np.diff(sign) != 0)[0] + 1
        runs = np.split(np.arange(grid), cuts)
        ext = np.array([r[np.argmax(np.abs(e[r]))] for r in runs if len(r)])
        if len(ext) != n:
            break
        new_ref = xs[ext]
        if np.allclose(new_ref, ref, rtol=0, atol=1e-12):
            break
        ref = new_ref
    return c, abs(E)


def kernel_error(coeffs32, n: int = 2000001) -> float:
    """Max relative error of the kernel's float32 evaluation (the Horner steps as float32
    fused multiply-adds, emulated in float64 with one rounding each) over f in [-1/2, 1/2]."""
    c0, c1, c2, c3 = (np.float64(np.float32(v)) for v in coeffs32)
    f = np.linspace(LO, HI, n).astype(np.float32).astype(np.float64)
    r32 = lambda v: v.astype(np.float32).astype(np.float64)
    p = r32(f * c3 + c2)
    p = r32(p * f + c1)
    p = r32(p * f + c0)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c, E = fit()
    c32 = [float(np.float32(v)) for v in c]
    print("c0..c3 =", ", ".join(f"{v:.10f}" for v in c32))
    print(f"levelled relative error {E:.3e}; float32 evaluation {kernel_error(c32):.3e}")
