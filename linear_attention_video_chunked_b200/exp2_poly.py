"""Coefficients of the FMA-pipe exp2 used for part of the softmax exponentials.

The attention kernel evaluates 2^x for a share of the logits on the FMA pipe
instead of the MUFU unit, using range reduction plus a polynomial:

    n = round(x)  (by adding and subtracting 1.5 * 2^23 in fp32),
    f = x - n in [-1/2, 1/2],
    2^x = 2^n * p(f),  with 2^n applied by adding n << 23 to the bits of p(f).

This is the classical split of Cody and Waite ("Software Manual for the
Elementary Functions", 1980) with the exponent-field construction described
by Schraudolph ("A fast, compact approximation of the exponential function",
Neural Computation, 1999).  p is a cubic fitted here: the coefficients
minimise the maximum relative error |p(f) / 2^f - 1| over a dense grid of
[-1/2, 1/2], solved exactly as a linear program, then rounded to fp32.

    python -m linear_attention_video_chunked_b200.exp2_poly

prints the coefficients (as fp32 hex and decimal) and the achieved maximum
relative error of the fp32 Horner evaluation; the kernel's constants must
equal them (tests/test_exp2_poly.py checks that).
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
GRID = 20001


def fit(degree: int = DEGREE, grid: int = GRID):
    """Minimax (discrete, relative error) polynomial for 2^f on [-1/2, 1/2]."""
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]  # p(f)/2^f
    # variables: c_0..c_d, e ; minimise e s.t. |V c - 1| <= e
    n = degree + 1
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -np.ones((grid, 1))]), np.hstack([-V, -np.ones((grid, 1))])])
    b = np.concatenate([np.ones(grid), -np.ones(grid)])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (n + 1), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return res.x[:n]


def as_fp32(coeffs):
    return np.asarray(coeffs, dtype=np.float64).astype(np.float32)


def horner_fp32(c32, f):
    """p(f) evaluated as the kernel does: fp32 FMA Horner."""
    f = np.asarray(f, np.float32)
    acc = np.full_like(f, c32[-1])
    for c in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f + np.float64(c)).astype(np.float32)  # fused: one rounding
    return acc


def emulate_exp2_fp32(c32, x):
    """Bit-level fp32 model of the kernel's exp2 for finite x in [-126, 126]."""
    x = np.asarray(x, np.float32)
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = horner_fp32(c32, f)
    n_bits = (t.view(np.uint32) << np.uint32(23)).astype(np.uint32)
    return (p.view(np.uint32) + n_bits).astype(np.uint32).view(np.float32)


def max_rel_error(c32, grid: int = 200001):
    f = np.linspace(-0.5, 0.5, grid).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(horner_fp32(c32, f).astype(np.float64) / ref - 1.0)))


def main():
    c32 = as_fp32(fit())
    for i, c in enumerate(c32):
        print(f"c{i} = {float(c)!r}  (0x{np.float32(c).view(np.uint32):08x})")
    print(f"max relative error (fp32 Horner on [-1/2, 1/2]): {max_rel_error(c32):.3e}")


if __name__ == "__main__":
    main()
