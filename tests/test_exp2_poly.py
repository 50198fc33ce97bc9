"""The forward kernel's FMA-pipe exp2 (exp2_fma_x2 in csrc/fwd_sm100.cu):
its cubic is the minimax fit of exp2_fit.py and its fp32 evaluation stays
within 2e-4 relative error of 2^x, far inside the bf16 rounding of P."""
import os
import re

import numpy as np

from attention_fwd_bwd_02_b200 import exp2_fit

SRC = os.path.join(os.path.dirname(exp2_fit.__file__), "csrc", "fwd_sm100.cu")


def _kernel_coeffs():
    src = open(SRC).read()
    start = src.index("exp2_fma_x2(")
    body = src[start:src.index("\n}\n", start)]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    vals = [v for v in vals if v < 2.0]  # drop the rounding constant
    # order in the source: c3, c2, c1, c0
    return [np.float32(v) for v in (vals[3], vals[2], vals[1], vals[0])]


def test_kernel_uses_the_fitted_coefficients():
    fitted = exp2_fit.coefficients_f32()
    kernel = _kernel_coeffs()
    for a, b in zip(fitted, kernel):
        assert abs(float(a) - float(b)) <= 2e-7 * abs(float(a)), (a, b)


def test_relative_error_bound_over_the_kernel_range():
    c = _kernel_coeffs()
    xs = np.linspace(-126.0, 8.0, 1000001).astype(np.float32)
    got = exp2_fit.emulate(xs, c).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 2e-4
    # integer points: the value of the cubic at f = 0 (and the boundary of
    # the normal range at -126)
    ints = np.arange(-126, 9, dtype=np.float32)
    assert np.all(np.abs(exp2_fit.emulate(ints, c) / np.exp2(ints.astype(np.float64)) - 1) < 2e-4)
