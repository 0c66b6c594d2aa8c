"""The FMA-pipe exp2 of the softmax (csrc/softmax_exp2.cuh): its polynomial
coefficients are the ones the fitting script in csrc/ produces, and their
fp32 Horner evaluation stays within the relative error the header states
(below fp16's half-ulp, 2^-12, the format P is stored in).  CPU only."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "diffusion_transformer_joint_attn_b200", "csrc")


def header_coefficients():
    text = open(os.path.join(CSRC, "softmax_exp2.cuh")).read()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = ([-+0-9.eE]+)f;", text))
    return [float(found[str(k)]) for k in range(len(found))]


def fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_coefficients_are_the_fitted_minimax_polynomial():
    coef = header_coefficients()
    fitted, _ = fit_module().fit(len(coef) - 1)
    assert len(coef) == 4                      # degree 3
    np.testing.assert_allclose(coef, fitted, rtol=1e-8, atol=0)


def test_fp32_evaluation_error_is_below_the_fp16_half_ulp():
    coef = header_coefficients()
    err = fit_module().fp32_horner_error(coef)
    assert err <= 7.6e-5                       # the bound the header states
    assert err < 2.0 ** -12                    # below fp16's half-ulp


def test_value_range_keeps_the_exponent_field_of_2_to_f():
    # the kernel adds j to the exponent field of p(f); p(f) in [0.70, 1.42]
    # keeps that field at 126 or 127 for every |f| <= 1/2
    coef = [np.float32(c) for c in header_coefficients()]
    f = np.linspace(-0.5, 0.5, 1 << 16, dtype=np.float32)
    p = np.full_like(f, coef[-1])
    for ck in reversed(coef[:-1]):
        p = (p.astype(np.float64) * f + np.float64(ck)).astype(np.float32)
    assert p.min() >= 0.70 and p.max() <= 1.42
    field = (p.view(np.uint32) >> 23) & 0xFF
    assert set(np.unique(field)) <= {126, 127}
