"""Fit the polynomial used by the kernel's FMA-pipe exp2 (build-time helper).

    python tiled_attention_18_b200/csrc/exp2_poly_fit.py [degree]

Method: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite style range reduction; n goes into the float's exponent
field), and 2^f approximated by the degree-d polynomial that minimises the
maximum relative error on [-1/2, 1/2], found with the Remez exchange
algorithm.  The script prints the coefficients (as float32, low order first)
and the maximum relative error of the float32-rounded coefficients
evaluated in float32 with Horner's rule.  The kernel hard-codes the printed
degree-3 values.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_relative(degree: int, a: float = -0.5, b: float = 0.5, iters: int = 30):
    """Minimax (relative error) polynomial for 2^x on [a, b]."""
    n = degree + 2  # reference points
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        f = np.exp2(x)
        # solve sum_j c_j x_i^j - f_i = (-1)^i E f_i   (relative error equioscillation)
        A = np.zeros((n, n))
        for j in range(degree + 1):
            A[:, j] = x ** j
        A[:, degree + 1] = -((-1.0) ** np.arange(n)) * f
        sol = np.linalg.solve(A, f)
        c, E = sol[:degree + 1], sol[degree + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sign[i] != sign[start]:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        if len(idx) < n:
            break
        # keep n points with the largest errors while preserving alternation
        idx = np.array(idx)
        while len(idx) > n:
            # drop the smaller end
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx = idx[1:]
            else:
                idx = idx[:-1]
        x = grid[idx]
    return c, abs(E)


def eval_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """Horner in float32 with fused multiply-add emulated in float64 then rounded."""
    p = np.full_like(f, c32[-1], dtype=np.float32)
    for cj in c32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(cj)).astype(np.float32)
    return p


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    degree = int(argv[0]) if argv else 3
    c, E = remez_relative(degree)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    p = eval_f32(c32, f)
    rel = np.abs(p.astype(np.float64) - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))
    print(f"degree {degree}: minimax relative error {E:.3e}; float32 evaluation max {rel.max():.3e}")
    for j, cj in enumerate(c32):
        print(f"  c{j} = {float(cj)!r}f  ({float(cj).hex()})")
    return 0


if __name__ == "__main__":
    sys.exit(main())
