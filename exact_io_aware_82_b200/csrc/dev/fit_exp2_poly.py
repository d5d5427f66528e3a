"""Fit the polynomial behind exp2_poly2 (dev/exp2_poly.cuh): 2^f on [-1/2, 1/2].

Method: the range reduction of Cody and Waite (x = j + f, j the integer nearest x, so that
2^x = 2^j * 2^f and 2^j is exact exponent arithmetic) leaves 2^f on [-1/2, 1/2], which a
polynomial of low degree approximates.  The coefficients minimise the largest RELATIVE error on
that interval, found by Lawson's algorithm (iteratively reweighted least squares, whose weights
converge to the minimax solution) on Chebyshev nodes, then rounded to fp32.

    python fit_exp2_poly.py [degree]    prints the coefficients and the fp32 error bound

The printed values are the ones the header holds; tests/test_exp2_poly.py refits and compares.
"""

from __future__ import annotations

import sys

import numpy as np


def fit(degree: int = 3, nodes: int = 4000, iters: int = 300) -> np.ndarray:
    """fp32 coefficients c[0..degree] (c[0] the constant term) of the minimax-relative fit."""
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)
    target = np.exp2(f)
    A = np.stack([f ** k for k in range(degree + 1)], axis=1) / target[:, None]
    w = np.full(nodes, 1.0 / nodes)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)[0]
        err = np.abs(A @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def exp2_poly_f32(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's sequence in fp32 arithmetic (round to nearest at every step): clamp,
    round-to-integer by adding 1.5 * 2^23, reduced argument, Horner, exponent added to the bits."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    fr = (x - j).astype(np.float32)
    p = np.full_like(fr, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * fr + c[k]).astype(np.float32)  # fma in the kernel: one rounding, not two
    bits = (t.view(np.uint32).astype(np.uint64) * (1 << 23) + p.view(np.uint32)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = fit(deg)
    xs = np.linspace(-30.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(exp2_poly_f32(xs, c).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)
    print("coefficients (constant term first):", ", ".join("%.9ef" % v for v in c))
    print("max relative error on [-30, 8] in fp32: %.3g" % rel.max())
