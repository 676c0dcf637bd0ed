"""The polynomial exp2 of the tensor-core kernel, modelled in float32 on the
CPU: its relative error bound over the inputs the kernel feeds it, and that the
coefficients compiled into the kernel are the ones checked here."""

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "h2o_kv_cache_attn_b200", "csrc")


def _mod():
    spec = importlib.util.spec_from_file_location("exp2_poly_coeffs",
                                                  os.path.join(CSRC, "exp2_poly_coeffs.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_relative_error_bound():
    m = _mod()
    assert m.max_rel_error(m.KERNEL_COEFFS) < 4e-6


def test_special_points():
    m = _mod()
    x = np.array([0.0, -1.0, -0.5, -0.25, -10.0, -126.0, -200.0, -np.inf], np.float32)
    y = m.exp2_poly(x, m.KERNEL_COEFFS)
    np.testing.assert_allclose(y[:6], np.exp2(x[:6].astype(np.float64)), rtol=4e-6)
    # clamped inputs give tiny non-negative values, never a wrapped exponent
    assert np.all(y[6:] >= 0) and np.all(y[6:] < 2.0 ** -125)


def test_kernel_uses_the_checked_coefficients():
    m = _mod()
    src = open(os.path.join(CSRC, "tc_ptx.cuh")).read()
    body = src[src.index("exp2_poly2"):]
    for c in m.KERNEL_COEFFS:
        assert re.search(re.escape(repr(float(c))) + "f", body), float(c)
