"""The polynomial the forward kernel uses for part of its exponentials.

ulysses_head_attention_b200/csrc/sm100.cuh evaluates 2^f on [-1/2, 1/2] as a
degree-3 polynomial whose coefficients come from fit_exp2_poly.py (Lawson's
iteratively reweighted least squares for the minimax relative error).  This
test re-runs the fit, checks that the coefficients written in sm100.cuh are
its output rounded to float32, and that they meet the stated error bound in
float32 Horner arithmetic, so the constants in the kernel cannot drift from
their derivation unnoticed.
"""
import importlib.util
import os
import re

import numpy as np

from conftest import ROOT

CSRC = os.path.join(ROOT, "ulysses_head_attention_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_kernel_constants_are_the_fit():
    m = _fit_module()
    c = m.fit(3)                                   # c0 + c1 f + c2 f^2 + c3 f^3
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = text[text.index("float exp2_poly(float x)"):]
    body = body[:body.index("return __int_as_float")]
    nums = [np.float32(float(x)) for x in re.findall(r"([0-9]+\.[0-9]+)f", body) if float(x) < 10.0]
    # Horner order in the kernel: c3, c2 (first fmaf), then c1, then c0
    assert nums == [np.float32(c[3]), np.float32(c[2]), np.float32(c[1]), np.float32(c[0])], (nums, c)


def test_fit_meets_its_error_bound_in_float32():
    m = _fit_module()
    c = m.fit(3)
    f = np.linspace(-0.5, 0.5, 200_001, dtype=np.float32)
    rel = np.abs(m.horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
