"""Fit the polynomial that the attention kernel uses for part of its exp2 work.

The softmax evaluates 2^x for every score.  The special-function unit that runs
``ex2.approx`` has a quarter of the FMA pipe's throughput on sm_100, so the kernel
evaluates a fraction of the exponentials on the FMA pipe instead, with the classical
range reduction

    x = n + f,  n = round-to-nearest-integer(x),  f in [-1/2, 1/2]
    2^x = 2^n * p(f)

where 2^n is applied by adding n to the float's exponent field and p is a polynomial
close to 2^f in *relative* error on [-1/2, 1/2].  This script computes p by the Remez
exchange algorithm (minimax relative error), rounds the coefficients to float32,
re-measures the error of a float32 Horner evaluation on a dense grid, and prints the
coefficients in the form pasted into attn_fwd.cuh.

Run:  python long_sequence_attention_b200/csrc/fit_exp2_poly.py [degree]
"""

import sys

import numpy as np


def remez_relative(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    """Minimax polynomial for 2^f on [lo, hi] with weight 1/2^f (relative error)."""
    n = degree + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: local extrema of the error, one per sign alternation
        sign = np.sign(err)
        idx = [0]
        for j in range(1, len(grid)):
            if sign[j] != sign[idx[-1]]:
                idx.append(j)
            elif abs(err[j]) > abs(err[idx[-1]]):
                idx[-1] = j
        idx = np.array(idx)
        if len(idx) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(idx) - n + 1), key=lambda s: np.min(np.abs(err[idx[s:s + n]])))
        x = grid[idx[best:best + n]]
    return coef


def f32_horner_error(coef32: np.ndarray, lo=-0.5, hi=0.5) -> float:
    f = np.linspace(lo, hi, 2000001).astype(np.float32)
    acc = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        acc = (acc * f + c).astype(np.float32)          # one fp32 fma per step (rounding of
    ref = 2.0 ** f.astype(np.float64)                    # a separate mul+add is close enough)
    return float(np.max(np.abs(acc.astype(np.float64) - ref) / ref))


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = remez_relative(degree)
    coef32 = coef.astype(np.float32)
    err = f32_horner_error(coef32)
    print(f"degree {degree}: max relative error (float32 Horner) = {err:.3e}")
    for i, c in enumerate(coef32):
        print(f"  c{i} = {float(c)!r}f  // bits 0x{np.float32(c).view(np.uint32):08x}")


if __name__ == "__main__":
    main()
