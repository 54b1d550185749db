"""The FMA-pipe exp2 used for part of the softmax exponentials: its constants are the ones the committed
fit produces, and the float32 evaluation (clamp, shifter rounding, Horner, exponent add) stays within its
error bound against exp2 over the whole input range the kernel feeds it."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_tiled_attention_43_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402


def header_constants():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    return np.array([float(re.search(rf"EXP2_C{k} = ([0-9.eE+-]+)f;", src).group(1)) for k in range(4)], np.float32)


def test_constants_match_the_fit():
    np.testing.assert_array_equal(header_constants(), fit_exp2_poly.fit())


def test_error_bound_over_kernel_range():
    c = header_constants()
    assert fit_exp2_poly.max_rel_error(c, -125.0, 8.0) < 1e-4
    # integers map to exact powers of two up to the polynomial's error at f = 0
    x = np.arange(-125, 9, dtype=np.float32)
    got = fit_exp2_poly.eval_f32(x, c).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4)
    # inputs below the clamp give 2^-125 (tiny, never garbage)
    y = fit_exp2_poly.eval_f32(np.array([-1e30, -300.0, -126.0], np.float32), c)
    assert np.all(y > 0) and np.all(y < 1e-37)
