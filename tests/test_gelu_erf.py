"""Pins of the erf approximation the CUDA kernels use inside GELU (host side).

The kernels evaluate erf by Hastings' formula as printed in Abramowitz and
Stegun, Handbook of Mathematical Functions, formula 7.1.28 (fixture
tests/golden/erf_hastings_7_1_28.json).  The tests read the constants compiled
into csrc/fno_common.cuh, check them against the printed ones, check the
printed error bound against SciPy's erf, and emulate in float32 the exact
operation sequence of the scalar and the paired (gelu2) GELU."""

import json
import os
import re

import numpy as np
from scipy.special import erf, erfc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "fourier_neural_spectral_fno_b200", "csrc", "fno_common.cuh")
GOLD = json.load(open(os.path.join(ROOT, "tests", "golden", "erf_hastings_7_1_28.json")))
F = np.float32


def _compiled_constants():
    text = open(HDR).read()
    return [float(re.search(r"kErfA%d = (-?\d+\.\d+(?:e-?\d+)?)f" % k, text).group(1))
            for k in range(1, 7)]


def _paired_constants():
    body = open(HDR).read().split("void erf_q16(")[1].split("f2unpack(q")[0]
    return [float(v) for v in re.findall(r"f2splat\((-?\d+\.\d+(?:e-?\d+)?)f\)", body)]


def _erfc_f32(t, coef):
    """The erfc half of gelu2, step by step in float32 (the reciprocal rounded
    once, as rcp.approx is within an ulp of it)."""
    t = F(t)
    q = F(coef[5]) * t + F(coef[4])
    for c in (coef[3], coef[2], coef[1], coef[0], 1.0):
        q = (q * t + F(c)).astype(F)
    for _ in range(4):
        q = (q * q).astype(F)
    with np.errstate(over="ignore", divide="ignore"):
        return (F(1) / q).astype(F)


def _erfc_pos_f32(t, coef):
    """erfc_pos step by step in float32: the power carried as v = q - 1."""
    t = F(t)
    u = F(coef[5]) * t + F(coef[4])
    for c in (coef[3], coef[2], coef[1], coef[0]):
        u = (u * t + F(c)).astype(F)
    u = (u * t).astype(F)
    with np.errstate(over="ignore", invalid="ignore"):
        for _ in range(4):
            u = (u * (u + F(2)).astype(F)).astype(F)
        return (F(1) / (F(1) + u).astype(F)).astype(F)


def test_compiled_constants_are_the_printed_ones():
    np.testing.assert_array_equal(F(_compiled_constants()), F(GOLD["a"]))


def test_printed_bound_holds_against_scipy():
    a = np.asarray(GOLD["a"])
    x = np.linspace(0.0, 12.0, 1_200_001)
    p = 1.0 + x * (a[0] + x * (a[1] + x * (a[2] + x * (a[3] + x * (a[4] + x * a[5])))))
    err = np.abs((1.0 - p ** -16.0) - erf(x))
    assert err.max() <= GOLD["max_abs_error"], err.max()


def test_a_dropped_or_altered_constant_breaks_the_bound():
    """The bound check above has teeth: each constant perturbed by 1 % (or the
    power 16 replaced by 15) violates it."""
    a0 = np.asarray(GOLD["a"])
    x = np.linspace(0.0, 6.0, 600_001)

    def worst(a, power=16.0):
        p = 1.0 + x * (a[0] + x * (a[1] + x * (a[2] + x * (a[3] + x * (a[4] + x * a[5])))))
        return np.abs((1.0 - p ** -power) - erf(x)).max()

    for k in range(6):
        a = a0.copy()
        a[k] *= 1.01
        assert worst(a) > GOLD["max_abs_error"], k
    assert worst(a0, 15.0) > GOLD["max_abs_error"]


def test_paired_constants_fold_one_over_sqrt2():
    """gelu2 takes |p| itself: its constants are a_k 2^(-k/2), highest first."""
    vals = _paired_constants()
    a = np.asarray(GOLD["a"])
    expect = [F(a[k] * 2.0 ** (-(k + 1) / 2.0)) for k in range(6)][::-1] + [F(1.0)]
    assert len(vals) == 7
    np.testing.assert_array_equal(F(vals), F(expect))


def test_scalar_norm_cdf_in_float32():
    a = _compiled_constants()
    p = np.linspace(-12.0, 12.0, 2_400_001).astype(F)
    t = (np.abs(p) * F(0.70710678118654752440)).astype(F)
    h = (F(0.5) * _erfc_pos_f32(t, a)).astype(F)
    cdf = np.where(p >= 0, F(1) - h, h).astype(np.float64)
    exact = 0.5 * erfc(-p.astype(np.float64) / np.sqrt(2.0))
    assert np.abs(cdf - exact).max() < 2.5e-7


def test_paired_gelu_in_float32():
    c = _paired_constants()[:6][::-1]      # lowest order first
    p = np.linspace(-12.0, 12.0, 2_400_001).astype(F)
    r = _erfc_f32(np.abs(p), c)
    w = (r * (p * F(0.5)).astype(F)).astype(F)
    g = np.where(p >= 0, (p - w).astype(F), w).astype(np.float64)
    pd = p.astype(np.float64)
    exact = 0.5 * pd * erfc(-pd / np.sqrt(2.0))
    err = np.abs(g - exact)
    assert (err / np.maximum(np.abs(pd), 1.0)).max() < 4.0e-7
    # zero and the far tails
    z = _erfc_f32(np.zeros(2, F), c) * F(0.0)
    assert np.all(z == 0.0)
    assert np.abs(g[pd < -9.0]).max() < 1e-15
    np.testing.assert_allclose(g[pd > 9.0], pd[pd > 9.0], rtol=1e-7, atol=0)


def test_doubled_paired_gelu_in_float32():
    """gelu2_dbl (the projection's activation, whose caller halves Q2): 2 GELU as
    2 p - p r or p r, step by step in float32."""
    c = _paired_constants()[:6][::-1]
    p = np.linspace(-12.0, 12.0, 2_400_001).astype(F)
    r = _erfc_f32(np.abs(p), c)
    w = (r * p).astype(F)
    g2 = np.where(p >= 0, (F(2) * p - w).astype(F), w).astype(np.float64)
    pd = p.astype(np.float64)
    exact = pd * erfc(-pd / np.sqrt(2.0))
    assert (np.abs(g2 - exact) / np.maximum(np.abs(pd), 1.0)).max() < 8.0e-7
    body = open(HDR).read().split("void gelu2_dbl(float &a, float &b)")[1].split("}")[0]
    assert "erf_q16(a, b, qa, qb)" in body and "fmaf(2.0f, a, -wa)" in body


def _grad_constants():
    body = open(HDR).read().split("void gelu_grad2(float &a, float &b)")[1].split("u = f2mul(u, t)")[0]
    return [float(v) for v in re.findall(r"f2splat\((-?\d+\.\d+(?:e-?\d+)?)f\)", body)]


def test_paired_gelu_grad_constants_match_the_paired_gelu():
    """gelu_grad2 folds 1 / sqrt 2 into the printed constants exactly as gelu2."""
    np.testing.assert_array_equal(F(_grad_constants()), F(_paired_constants()[:6]))


def test_paired_gelu_grad_in_float32():
    """GELU'(p) = Phi(p) + p phi(p), step by step as gelu_grad2: Phi through the
    q - 1 form (the reciprocal rounded once), phi through 2^(-p^2 log2(e) / 2)
    (the power of two evaluated exactly, then rounded, as ex2.approx is within
    2^-22 of it)."""
    c = _grad_constants()[::-1]           # lowest order first
    p = np.linspace(-12.0, 12.0, 2_400_001).astype(F)
    h = (F(0.5) * _erfc_pos_f32(np.abs(p), c)).astype(F)
    cdf = np.where(p >= 0, (F(1) - h).astype(F), h)
    ex = ((p * p).astype(F) * F(-0.72134752044448170368)).astype(F)
    phi = (np.exp2(ex.astype(np.float64)).astype(F) * F(0.39894228040143267794)).astype(F)
    got = (p.astype(np.float64) * phi + cdf).astype(F).astype(np.float64)
    pd = p.astype(np.float64)
    exact = 0.5 * erfc(-pd / np.sqrt(2.0)) + pd * np.exp(-0.5 * pd * pd) / np.sqrt(2.0 * np.pi)
    assert np.abs(got - exact).max() < 4.0e-7
