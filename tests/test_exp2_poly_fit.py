"""The software 2^x of the prefill softmax, checked on the host.

The coefficients in ptx_sm100.cuh must be the ones csrc/fit_exp2_poly.py fits
(a discrete minimax problem solved as a linear program), and the evaluation
scheme (Cody & Waite reduction x = n + f with the 1.5 * 2^23 rounding constant,
Horner in f, n added to the exponent field) replayed step by step in float32
with numpy must stay within the fitted relative error over the range the
softmax uses, and give exactly 0 below 2^-126.  The device version is checked
against the same bound by tests/test_exp2_poly_gpu.py.
"""

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attention_tiled_attn_b200", "csrc")


def _header_constants():
    text = open(os.path.join(CSRC, "ptx_sm100.cuh")).read()
    get = lambda n: float(re.search(rf"constexpr float {n} = ([-0-9.eE+]+)f;", text).group(1))  # noqa: E731
    return np.float32([get("EXP2_C1"), get("EXP2_C2"), get("EXP2_C3")]), np.float32(get("ROUND_MAGIC"))


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _exp2_scheme(x, c, magic):
    """Float32 replay of the device scheme, one rounding per operation as the FMAs do."""
    x = np.float32(x)
    zero = x < np.float32(-126.0)
    with np.errstate(invalid="ignore", over="ignore"):
        t = (x.astype(np.float64) + np.float64(magic)).astype(np.float32)      # x + M, rounded once
        n = (t.astype(np.float64) - np.float64(magic)).astype(np.float32)      # exact
        f = (x.astype(np.float64) - n.astype(np.float64)).astype(np.float32)   # exact
        q = (f.astype(np.float64) * c[2] + c[1]).astype(np.float32)
        q = (q.astype(np.float64) * f + c[0]).astype(np.float32)
        q = (q.astype(np.float64) * f + 1.0).astype(np.float32)
        bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return np.where(zero, np.float32(0.0), bits.view(np.float32))


def test_header_constants_are_the_fitted_ones():
    c, magic = _header_constants()
    coef, err = _fit_module().fit()
    assert np.array_equal(coef, c), (coef, c)
    assert magic == np.float32(1.5 * 2 ** 23)
    assert err < 1.05e-4


def test_scheme_relative_error_and_flush():
    c, magic = _header_constants()
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001), np.float32([-0.5, 0.5, -125.5, 7.5])]).astype(np.float32)
    y = _exp2_scheme(x, c, magic)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) / ref - 1.0)
    assert rel.max() < 1.1e-4, rel.max()
    below = np.float32([-126.001, -127.0, -150.0, -1e30, -np.inf])
    assert np.all(_exp2_scheme(below, c, magic) == 0.0)
