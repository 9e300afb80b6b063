"""Coefficients of the FMA-pipe 2^x in ptx.cuh (ex2_fma2).

After Cody-Waite range reduction x = j + f (j = round(x), f in [-1/2, 1/2]), 2^f is
replaced by the polynomial of the given degree whose largest RELATIVE error on
[-1/2, 1/2] is smallest. The polynomial is found by the Remez exchange algorithm:
solve for the polynomial that equioscillates with equal weighted error on a reference
set of deg + 2 points, move the reference to the extrema of the new error curve, and
repeat until the reference stops moving. The coefficients are then rounded to float32
and the polynomial re-evaluated in float32 Horner form, which is how the kernel runs it.

    python fit_exp2_poly.py [degree]     # prints the float32 coefficients, c0 first
"""

import sys

import numpy as np


def remez_exp2(degree, a=-0.5, b=0.5, iterations=40, grid=200001):
    """Minimax-relative-error polynomial for 2^f on [a, b]; returns (coeffs c0.., error)."""
    n = degree + 2
    # start from the Chebyshev extrema mapped onto [a, b]
    ref = 0.5 * (a + b) - 0.5 * (b - a) * np.cos(np.pi * np.arange(n) / (n - 1))
    g = np.linspace(a, b, grid)
    coeffs, err_max = None, None
    for _ in range(iterations):
        target = 2.0 ** ref
        # p(ref_i) - 2^ref_i = (-1)^i E 2^ref_i, unknowns: the coefficients and E
        system = np.zeros((n, n))
        system[:, : degree + 1] = ref[:, None] ** np.arange(degree + 1)[None, :]
        system[:, degree + 1] = (-1.0) ** np.arange(n) * target
        sol = np.linalg.solve(system, target)
        coeffs = sol[: degree + 1]
        err = np.polynomial.polynomial.polyval(g, coeffs) / 2.0 ** g - 1.0
        err_max = float(np.max(np.abs(err)))
        # one extremum of |err| per run of constant sign
        edges = np.concatenate(([0], np.nonzero(np.diff(np.sign(err)))[0] + 1, [grid]))
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(edges[:-1], edges[1:]) if hi > lo]
        if len(ext) != n:
            break
        new_ref = g[ext]
        if np.allclose(new_ref, ref, rtol=0, atol=1e-12):
            break
        ref = new_ref
    return coeffs, err_max


def float32_horner_error(coeffs32, a=-0.5, b=0.5, grid=100001):
    """Largest relative error of the float32 coefficients evaluated in float32 Horner form."""
    f = np.linspace(a, b, grid).astype(np.float32)
    p = np.full_like(f, coeffs32[-1])
    for c in coeffs32[-2::-1]:
        p = (p * f + c).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


def fit(degree=4):
    coeffs, err = remez_exp2(degree)
    c32 = coeffs.astype(np.float32)
    return c32, err, float32_horner_error(c32)


if __name__ == "__main__":
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c32, err, err32 = fit(degree)
    for k, c in enumerate(c32):
        print("kC%d = %.17gf" % (k, float(c)))
    print("minimax relative error %.3e, float32 Horner %.3e" % (err, err32))
