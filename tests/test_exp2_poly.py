"""The FMA-pipe exponential of the prefill softmax (dev/exp2_poly.cuh), checked on the CPU.

- the coefficients in the header are those the fitting script computes (Lawson's minimax fit of
  2^f on [-1/2, 1/2]), to fp32;
- the kernel's sequence of fp32 steps, replayed in numpy, stays within 1e-4 relative of 2^x over
  the range where a weight can matter (-125 <= x <= 8; the running sum it joins is at least 1),
  far inside the 2^-9 relative rounding of the bf16 weights it produces, and below that it
  gives non-negative values under 2^-125 (the clamp at -126 keeps the exponent in its field);
- the range reduction is exact at integers (2^j comes out as a power of two times c0).
"""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEV = os.path.join(ROOT, "exact_io_aware_82_b200", "csrc", "dev")
sys.path.insert(0, DEV)

import fit_exp2_poly as F  # noqa: E402


def header_coefficients():
    with open(os.path.join(DEV, "exp2_poly.cuh")) as fh:
        text = fh.read()
    vals = dict(re.findall(r"constexpr float kExp2C(\d) = ([-+0-9.e]+)f;", text))
    return np.array([float(vals[str(k)]) for k in range(4)], dtype=np.float32)


def test_header_holds_the_fitted_coefficients():
    c = header_coefficients()
    fitted = F.fit(3)
    assert np.allclose(c, fitted, rtol=2e-7, atol=0), (c, fitted)


def test_relative_error_bound_over_the_softmax_range():
    c = header_coefficients()
    xs = np.concatenate([np.linspace(-125.0, 8.0, 4_000_001, dtype=np.float32),
                         np.float32(np.arange(-125, 9))])
    got = F.exp2_poly_f32(xs, c).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4, rel.max()
    # and the bf16 rounding that follows dominates it by more than an order of magnitude
    assert rel.max() < 2.0 ** -9 / 10


def test_integers_are_powers_of_two_times_c0():
    c = header_coefficients()
    j = np.arange(-125, 9).astype(np.float32)
    got = F.exp2_poly_f32(j, c).astype(np.float64)
    assert np.array_equal(got, np.exp2(j.astype(np.float64)) * np.float64(c[0]))


def test_clamp_keeps_the_sign_and_exponent_sane():
    c = header_coefficients()
    got = F.exp2_poly_f32(np.array([-np.inf, -1e30, -300.0, -127.0, -126.0, -125.5], np.float32), c)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -125)
