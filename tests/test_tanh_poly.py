"""The FMA-pipe tanh used for part of HSTU's pointwise step: its constants are the ones the committed fit
produces, and its float32 evaluation stays within the fit's error bound against tanh on [-1, 1], the only
range the kernel feeds it (tighter than the MUFU's tanh.approx, whose relative error is about 2^-11)."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_tiled_attention_43_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_tanh_poly  # noqa: E402


def header_constants():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    return np.array([float(re.search(rf"TANH_C{k} = ([0-9.eE+-]+)f;", src).group(1)) for k in range(4)],
                    np.float32)


def test_constants_match_the_fit():
    np.testing.assert_array_equal(header_constants(), fit_tanh_poly.fit())


def test_error_bound_on_the_kernel_range():
    c = header_constants()
    assert fit_tanh_poly.max_abs_error(c) < 4e-5
    # odd: tanh(-y) = -tanh(y) exactly in the float32 evaluation, and tanh(0) = 0
    y = np.linspace(0, 1, 1001, dtype=np.float32)
    np.testing.assert_array_equal(fit_tanh_poly.eval_f32(-y, c), -fit_tanh_poly.eval_f32(y, c))
    assert fit_tanh_poly.eval_f32(np.zeros(1, np.float32), c)[0] == 0.0
    # the end point: tanh(1) = 0.7615941559557649
    assert abs(float(fit_tanh_poly.eval_f32(np.ones(1, np.float32), c)[0]) - 0.7615941559557649) < 4e-5
