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
    found = {int(i): np.float32(float(v)) for i, v in re.findall(r"kExp2PolyC([0-3]) = ([0-9]+\.[0-9]+)f;", text)}
    assert found == {i: np.float32(c[i]) for i in range(4)}, (found, c)
    # both the scalar and the packed evaluation use the named constants, in Horner order
    for fn in ("float exp2_poly(float x)", "uint64_t exp2_poly2(uint64_t x2)"):
        body = text[text.index(fn):]
        body = body[:body.index("return ")]
        assert not re.findall(r"0\.[0-9]{5,}f", body), fn
        order = [int(x) for x in re.findall(r"kExp2PolyC([0-3])", body)]
        assert [x for i, x in enumerate(order) if i == 0 or x != order[i - 1]] == [3, 2, 1, 0], (fn, order)


def test_fit_meets_its_error_bound_in_float32():
    m = _fit_module()
    c = m.fit(3)
    f = np.linspace(-0.5, 0.5, 200_001, dtype=np.float32)
    rel = np.abs(m.horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
