"""The FMA-pipe exp2 of the attention kernel (csrc/tc_common.cuh,
exp2_poly2): its constants equal a fresh minimax fit, and a bit-level fp32
model of it stays within the stated relative error of 2^x.

Method: range reduction to f = x - round(x) in [-1/2, 1/2] (Cody and Waite,
1980), a cubic for 2^f fitted here for minimax relative error, and 2^n
applied through the exponent field (Schraudolph, 1999).  The error bound
(1e-4 relative) is well below bf16's half-ulp (2^-9), the rounding P gets
before the P.V product.
"""
import os
import re

import numpy as np
import pytest

from linear_attention_video_chunked_b200 import exp2_poly

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "linear_attention_video_chunked_b200", "csrc", "tc_common.cuh")


def _kernel_coeffs():
    text = open(HEADER).read()
    found = dict(re.findall(r"k(C\d) = ([0-9.eE+-]+)f", text))
    return np.array([float(found[f"C{i}"]) for i in range(4)], dtype=np.float32)


def test_kernel_constants_equal_the_fit():
    fitted = exp2_poly.as_fp32(exp2_poly.fit())
    np.testing.assert_array_equal(_kernel_coeffs(), fitted)


def test_relative_error_bound_on_reduced_range():
    assert exp2_poly.max_rel_error(_kernel_coeffs()) < 1e-4


@pytest.mark.parametrize("lo,hi", [(-125.0, -100.0), (-30.0, 0.0), (-1.0, 1.0), (0.0, 8.0)])
def test_bit_level_model_against_exp2(lo, hi):
    x = np.linspace(lo, hi, 100001).astype(np.float32)
    got = exp2_poly.emulate_exp2_fp32(_kernel_coeffs(), x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4


def test_exact_at_integers_up_to_the_polynomial_error():
    x = np.arange(-125, 9, dtype=np.float32)
    got = exp2_poly.emulate_exp2_fp32(_kernel_coeffs(), x).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4)
