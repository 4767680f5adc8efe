"""The polynomial 2^x used for part of the prefill softmax: the committed
coefficients are the fit that csrc/exp2_poly.py computes, and the float32
instruction sequence stays within its relative error bound over the range
the kernel feeds it (x <= 8 after the lazy-rescale reference, far below 0
for masked or negligible terms)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "differential_attention_sm_b200", "csrc")


def _load_fit():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_header_constants_match_fit():
    m = _load_fit()
    coef, err = m.fit()
    assert err < 1e-4
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    got = [float(v) for v in re.findall(r"kExp2C(\d) = ([-0-9.e+]+)f;", text) and
           [x[1] for x in sorted(re.findall(r"kExp2C(\d) = ([-0-9.e+]+)f;", text))]]
    assert len(got) == 4
    assert np.allclose(got, np.float32(coef), rtol=1e-7, atol=0)


def test_float32_sequence_error_bound():
    m = _load_fit()
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    coef = [float(x[1]) for x in sorted(re.findall(r"kExp2C(\d) = ([-0-9.e+]+)f;", text))]
    xs = np.linspace(-100.0, 8.0, 400001, dtype=np.float32)
    got = m.emulate_fp32(xs, coef).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    keep = xs > -125.0
    assert np.abs(got[keep] / ref[keep] - 1.0).max() < 1e-4
    # clamped region: tiny and non-negative
    assert (got[~keep] >= 0).all() and (got[~keep] < 1e-37).all()
