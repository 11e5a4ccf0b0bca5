"""The worst-case score error of the tensor-core read's fixed-point digits, for
every head width and bit count that kernel serves (CPU only).

tests/digit_split.py restates the split (centroid digits hi/lo, query digits
D0..D2) from its definition and bounds the error over all queries and codes.
The bound must stay inside the 1e-4 * ||q|| ||k|| / sqrt(d) score tolerance for
every (d, b).  The GPU test tests/test_read_worst_case_gpu.py runs the case
that reaches the centroid term of the bound and checks the kernel against both.
"""
import numpy as np
import pytest

import digit_split
from lut_attention_b200 import axr

WIDTHS = (128, 256, 512)


@pytest.fixture(scope="module")
def lib(axr_lib):
    return axr_lib


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", WIDTHS)
def test_digits_represent_the_centroids(lib, d, b):
    cent, _ = axr.axr_make_codebook(d, b)
    hi, lo, v, cmax = digit_split.centroid_digits(cent)
    assert np.all(np.abs(hi) <= 127) and np.all(np.abs(lo) <= 64)
    assert np.all(128 * hi + lo == v)
    assert np.abs(v).max() == 128 * 127                       # the largest centroid maps to 127 * 128
    err = digit_split.centroid_errors(cent)
    assert np.abs(err).max() <= 0.5 * cmax / (128 * 127) * (1 + 1e-12)
    # a symmetric codebook gives antisymmetric digits
    assert np.array_equal(hi, -hi[::-1]) and np.array_equal(lo, -lo[::-1])


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", WIDTHS)
def test_worst_case_bound_is_inside_the_tolerance(lib, d, b):
    cent, _ = axr.axr_make_codebook(d, b)
    bound, M = digit_split.worst_case_bound(cent, d)
    _, aligned = digit_split.aligned_worst_case(cent, d)
    # the aligned case reaches the centroid term of the bound at M = 1/sqrt(d)
    assert abs(aligned) <= bound
    # fp32 steps of the kernel (rotation, conversions, the final scale) add < 1e-6
    assert bound + 1e-6 <= 1e-4, f"d={d} b={b}: worst case {bound:.3e} at M={M:.3f}"


def test_bound_depends_on_bits_not_width(lib):
    """The centroid term sqrt(d) * dc is a property of the standard-normal
    codebook (c ~ 1/sqrt(d)), so the same b gives the same aligned error at
    every width, to fp32 rounding of the centroids."""
    for b in (1, 2, 3, 4):
        vals = [digit_split.aligned_worst_case(axr.axr_make_codebook(d, b)[0], d)[1] for d in WIDTHS]
        assert max(abs(v) for v in vals) - min(abs(v) for v in vals) < 1e-7, (b, vals)
