"""Pins of the erf polynomial the CUDA kernels use inside GELU (host side):
the generator reproduces the coefficients compiled into the kernels, and the
float32 Horner evaluation stays within 6e-7 of the double-precision erf."""

import os
import re

import numpy as np
from scipy.special import erf

from fourier_neural_spectral_fno_b200 import gen_erf_poly

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "fourier_neural_spectral_fno_b200", "csrc", "fno_common.cuh")


def _compiled_coefficients():
    body = open(HDR).read().split("erf_pos(float t)")[1].split("return")[0]
    vals = re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body)
    return [float(v) for v in vals[3:]]   # skip 3.9, 1.95, 1/1.95 of the variable change


def test_generator_reproduces_compiled_coefficients():
    coef = gen_erf_poly.fit()
    compiled = _compiled_coefficients()
    assert len(compiled) == gen_erf_poly.DEGREE + 1
    np.testing.assert_allclose(np.float32(coef[::-1]), np.float32(compiled), rtol=0, atol=0)


def test_float32_evaluation_accuracy():
    coef = np.asarray(_compiled_coefficients()[::-1], np.float64)
    t = np.linspace(0.0, 8.0, 400001)
    err = np.max(np.abs(gen_erf_poly.eval_f32(coef, t) - erf(t)))
    assert err < 6e-7, err


def test_gelu_from_polynomial_matches_exact_gelu():
    coef = np.asarray(_compiled_coefficients()[::-1], np.float64)
    p = np.linspace(-9.0, 9.0, 200001)
    e = gen_erf_poly.eval_f32(coef, np.abs(p) / np.sqrt(2.0)).astype(np.float64)
    gelu = p * (0.5 + 0.5 * np.sign(p) * e)
    exact = 0.5 * p * (1.0 + erf(p / np.sqrt(2.0)))
    assert np.max(np.abs(gelu - exact)) < 3e-7
    big = np.abs(exact) > 0.1          # away from the cancelling negative tail
    assert np.max(np.abs(gelu - exact)[big] / np.abs(exact)[big]) < 2e-6


def test_paired_gelu_matches_scalar_coefficients():
    """The paired GELU (gelu2) evaluates the same polynomial as erf_pos: its
    f2splat literals are the scalar coefficients, preceded by the variable
    change x = |p| / (1.95 sqrt 2) - 1 (the scale to float32 rounding)."""
    body = open(HDR).read().split("void gelu2(float &a, float &b)")[1].split("f2unpack(e")[0]
    vals = [float(v) for v in re.findall(r"f2splat\((-?\d+\.\d+(?:e-?\d+)?)f\)", body)]
    assert len(vals) == 2 + gen_erf_poly.DEGREE + 1
    assert np.float32(vals[0]) == np.float32(1.0 / (1.95 * np.sqrt(2.0)))
    assert vals[1] == -1.0
    np.testing.assert_array_equal(np.float32(vals[2:]), np.float32(_compiled_coefficients()))
