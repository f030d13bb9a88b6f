"""The cubic the prefill kernel uses for part of its exp2 work: its
coefficients are the ones the committed fit produces, and its relative error
(fp32 Horner evaluation, as on the GPU) stays far below bf16 resolution."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "decode_swa_prefill_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402


def kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = src[src.index("float2 exp2_poly2"):]
    body = body[:body.index("float2 r;")]
    vals = re.findall(r"make_float2\(([0-9.e+-]+)f, \1f\)", body)
    # skip the rounding constants; keep the four polynomial coefficients
    return [float(v) for v in vals if abs(float(v)) < 2.0 and float(v) != -1.0]


def test_kernel_uses_the_fitted_cubic():
    c = fit_exp2_poly.fit(3).astype(np.float32)
    assert np.allclose(kernel_coefficients(), c, rtol=1e-6, atol=0)


def test_relative_error_far_below_bf16():
    err = fit_exp2_poly.max_rel_error(fit_exp2_poly.fit(3))
    assert err < 1e-4          # bf16 half-ulp is 2^-9 ~ 2e-3


def test_range_reduction_reconstructs_powers_of_two():
    # integer arguments: the fraction is 0, so the result is 2^j * p(0)
    c = fit_exp2_poly.fit(3)
    for j in (-125, -20, -1, 0, 1, 5, 8):
        p0 = np.float32(c[-1])
        val = np.frombuffer((np.frombuffer(p0.tobytes(), np.int32) + (j << 23)).astype(np.int32).tobytes(),
                            np.float32)[0]
        assert abs(val / 2.0 ** j - 1) < 1e-4
