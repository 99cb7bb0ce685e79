"""The FMA-pipe exp2 used for part of the softmax: its coefficients are the
committed fit's, and its float32 arithmetic stays within the fit's error bound
over the range the softmax feeds it (running-max-relative logits)."""

import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "dynamic_hierarchical_sparse_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly_fit  # noqa: E402


def _header_coefficients():
    with open(os.path.join(CSRC, "exp2_poly.cuh")) as f:
        text = f.read()
    c = [float(x) for x in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", text)]
    # Horner order in the header: c3, c2, c1, c0
    return [c[3], c[2], c[1], c[0]]


def test_header_matches_fit():
    coef, err = exp2_poly_fit.fit()
    assert err < 8e-5
    np.testing.assert_allclose(_header_coefficients(), coef, rtol=2e-9)


def test_float32_emulation_error_bound():
    coef = _header_coefficients()
    xs = np.concatenate([np.linspace(-125, 8.5, 400001), np.arange(-40, 9, 0.5)]).astype(np.float32)
    got = exp2_poly_fit.emulate_f32(xs, coef).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1)
    assert rel.max() < 8e-5
    # clamped tail: far below any softmax weight that survives bf16 rounding
    tail = exp2_poly_fit.emulate_f32(np.array([-200.0, -1e30, -np.inf], dtype=np.float32), coef)
    assert np.all(tail >= 0) and np.all(tail < 1e-37)
