"""The approximation constants written in the kernels' source, checked on the
CPU (float64) against the mathematics they approximate, so that a mistyped
coefficient fails here without a GPU (the -m gpu tests then check the
compiled functions themselves):

* the GEMM epilogue's GELU (scalar and packed forms): the normal tail
  probability by the rational approximation 7.1.26 of Abramowitz and Stegun,
  whose published coefficients are halved in the source; within the
  approximation's error bound of the exact GELU;
* the attention softmax's FMA-pipe 2^x: a degree-3 polynomial on the
  reduced argument, within its stated relative error of 7.5e-5.
"""
import os
import re

import numpy as np
from scipy.special import erfc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "flow_matching_video_b200", "csrc")

# Abramowitz and Stegun 7.1.26 (Hastings): erf(y) = 1 - t (a1 + t (a2 + ...)) exp(-y^2), t = 1 / (1 + p y)
AS_P = 0.3275911
AS_A = (0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429)


def _function_body(path, signature):
    src = open(os.path.join(CSRC, path), encoding="utf-8").read()
    i = src.index(signature)
    j = src.index("\n}", i)
    return src[i:j]


def _floats(text):
    return [float(v) for v in re.findall(r"(-?\d+\.\d+)f", text)]


def _gelu_constants(signature):
    body = _function_body("wd_internal.cuh", signature)
    vals = _floats(body)
    # 1/sqrt(2), p, 1, -log2(e), then the polynomial innermost first (a5/2 ... a1/2)
    inv_sqrt2 = next(v for v in vals if abs(v - 0.7071) < 1e-3)
    p = next(v for v in vals if abs(v - 0.3276) < 1e-3)
    neg_log2e = next(v for v in vals if abs(v + 1.4427) < 1e-3)
    poly = [v for v in vals if any(abs(v - a / 2) < 1e-3 for a in AS_A)]
    return inv_sqrt2, p, neg_log2e, poly


def _gelu_from(consts, x):
    inv_sqrt2, p, neg_log2e, poly = consts
    y = np.abs(x) * inv_sqrt2
    t = 1.0 / (1.0 + p * y)
    acc = np.full_like(t, poly[0])
    for c in poly[1:]:
        acc = acc * t + c
    tail = t * acc * np.exp2(neg_log2e * y * y)
    return x * np.where(x >= 0, 1.0 - tail, tail)


def test_gelu_constants_are_the_published_ones_halved():
    for sig in ("float gelu_as(float x)", "float2 gelu_as2(float2 x)"):
        inv_sqrt2, p, neg_log2e, poly = _gelu_constants(sig)
        assert abs(inv_sqrt2 - 1 / np.sqrt(2.0)) < 1e-15 and abs(neg_log2e + 1 / np.log(2.0)) < 1e-15
        assert p == AS_P
        assert len(poly) == 5
        np.testing.assert_allclose([2 * c for c in reversed(poly)], AS_A, rtol=0, atol=1e-9)


def test_gelu_formula_within_its_bound_of_the_exact_gelu():
    """The published bound |erf error| <= 1.5e-7 moves x Phi(x) by at most
    0.75e-7 |x|; the source's formula (in float64) stays inside it."""
    x = np.linspace(-30.0, 30.0, 600_001)
    exact = 0.5 * x * erfc(-x / np.sqrt(2.0))
    for sig in ("float gelu_as(float x)", "float2 gelu_as2(float2 x)"):
        got = _gelu_from(_gelu_constants(sig), x)
        assert np.all(np.abs(got - exact) <= 0.75e-7 * np.abs(x) + 1e-15), sig


def test_exp2_polynomial_within_its_stated_relative_error():
    """x = j + f with j = round(x), |f| <= 1/2; 2^x = q(f) 2^j with q the
    source's degree-3 polynomial: relative error at most 7.5e-5, the bound
    stated beside it; the scalar and packed forms carry the same coefficients."""
    forms = []
    for sig in ("float exp2_fma(float x)", "float2 exp2_fma2(float2 x)"):
        body = _function_body("k_attn_tc.cu", sig)
        coeffs = []
        for v in _floats(body):   # the packed form writes each coefficient twice (both lanes)
            if abs(v) < 2.0 and v not in coeffs:
                coeffs.append(v)
        forms.append(coeffs)
    assert forms[0] == forms[1] and len(forms[0]) == 4
    c3, c2, c1, c0 = forms[0]
    f = np.linspace(-0.5, 0.5, 200_001)
    q = ((c3 * f + c2) * f + c1) * f + c0
    assert np.abs(q / np.exp2(f) - 1.0).max() <= 7.5e-5
