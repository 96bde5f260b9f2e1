"""The exponential polynomial the kernels use is the Remez fit that
fit_exp2_poly.py computes: the coefficients written in tc_primitives.cuh
(scalar and packed forms) equal the fit's float32 values, and the fit meets
its stated bound.  CPU only."""
import os
import re

import numpy as np

from rank_latent_attention_flare_b200 import fit_exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "rank_latent_attention_flare_b200", "csrc", "tc_primitives.cuh")


def _header_coeffs():
    text = open(HDR).read()
    sets = []
    for m in re.finditer(r"constexpr float kE0 = ([-\d.e]+)f, kE1 = ([-\d.e]+)f;\s*"
                         r"constexpr float kE2 = ([-\d.e]+)f, kE3 = ([-\d.e]+)f;", text):
        sets.append([float(v) for v in m.groups()])
    return sets


def test_header_coefficients_are_the_fit():
    c, err = fit_exp2_poly.remez_exp2()
    c32 = [float(np.float32(v)) for v in c]
    sets = _header_coeffs()
    assert len(sets) == 3, "expected the scalar, packed and clamped packed polynomials"
    for s in sets:
        assert [float(np.float32(v)) for v in s] == c32
    assert err <= 7.5e-5


def test_fit_is_minimax_equioscillating():
    # the relative error of the fit equioscillates at deg + 2 points with
    # the maximum magnitude (the Remez optimality condition)
    c, err = fit_exp2_poly.remez_exp2()
    f = np.linspace(-0.5, 0.5, 200001)
    e = np.polyval(np.asarray(c)[::-1], f) / np.exp2(f) - 1.0
    peaks = []
    for i in range(1, f.size - 1):
        if abs(e[i]) >= abs(e[i - 1]) and abs(e[i]) >= abs(e[i + 1]) and abs(e[i]) > 0.99 * err:
            peaks.append(np.sign(e[i]))
    ends = [np.sign(e[0])] if abs(e[0]) > 0.99 * err else []
    ends += [np.sign(e[-1])] if abs(e[-1]) > 0.99 * err else []
    signs = ends[:1] + peaks + ends[1:]
    assert len(signs) >= 5
    assert all(a != b for a, b in zip(signs, signs[1:]))
