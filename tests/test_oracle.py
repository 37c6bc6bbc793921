"""Pins of the CPU oracle against things other than itself.

Each test would fail under a plausible slip in the oracle: a dropped term, a
wrong sign or index, a transposed operand, a wrong normalisation or mode
weight.  Sources: hand-derived fixtures in tests/golden (with their
derivations), closed forms of single-mode inputs, Parseval's identity, the
all-modes identity, brute-force d-dimensional sums, NumPy's FFT as an
independent library routine, adjoint identities and finite differences.
"""

import json
import os

import numpy as np
import pytest

import oracle as O
from fourier_neural_spectral_fno_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_r(rng, ci, co, k):
    return rng.standard_normal((ci, co, k)) + 1j * rng.standard_normal((ci, co, k))


# --------------------------------------------------------------------------
# hand-derived fixtures
# --------------------------------------------------------------------------

def test_golden_1d_block_forward_and_backward():
    g = _load("block1d_n4_hand.json")
    x = np.array(g["x"]).reshape(1, 1, 4)
    r = (np.array(g["R_re"]) + 1j * np.array(g["R_im"])).reshape(1, 1, -1)
    y, xhat = O.spectral_conv_fwd(x, r, g["modes"])
    np.testing.assert_allclose(xhat.ravel(), np.array(g["xhat_re"]) + 1j * np.array(g["xhat_im"]),
                               atol=1e-12)
    np.testing.assert_allclose(y.ravel(), g["y_spec"], atol=1e-12)
    _, pre, _ = O.block_fwd(x, r, np.array(g["W"]), np.array(g["b"]), g["modes"])
    np.testing.assert_allclose(pre.ravel(), g["pre"], atol=1e-12)
    dx, d_r = O.spectral_conv_bwd(x, r, xhat, np.array(g["dy"]).reshape(1, 1, 4), g["modes"])
    np.testing.assert_allclose(dx.ravel(), g["dx_spec"], atol=1e-12)
    np.testing.assert_allclose(d_r.ravel(), np.array(g["dR_re"]) + 1j * np.array(g["dR_im"]),
                               atol=1e-12)


def test_golden_2d_block():
    g = _load("block2d_2x2_hand.json")
    x = np.array(g["x"]).reshape(1, 1, 2, 2)
    r = (np.array(g["R_re"]) + 1j * np.array(g["R_im"])).reshape(1, 1, -1)
    y, xhat = O.spectral_conv_fwd(x, r, g["modes"])
    np.testing.assert_allclose(xhat.ravel(), np.array(g["xhat_re"]) + 1j * np.array(g["xhat_im"]),
                               atol=1e-12)
    np.testing.assert_allclose(y.reshape(2, 2), g["y_spec"], atol=1e-12)


def test_golden_network_composition():
    g = _load("network_scalar_hand.json")
    grid, modes = tuple(g["grid"]), tuple(g["modes"])
    nk = O.num_modes(grid, modes)
    params = {"P": np.array([[g["P"]]]), "p": np.array([g["p"]]),
              "R": [np.zeros((1, 1, nk), complex)], "W": [np.array([[g["W"]]])],
              "b": [np.array([g["b"]])], "Q1": np.array([[g["Q1"]]]), "q1": np.array([g["q1"]]),
              "Q2": np.array([[g["Q2"]]]), "q2": np.array([g["q2"]])}
    a = np.full((1, 1) + grid, g["a"])
    np.testing.assert_allclose(O.forward(a, params, modes), np.full((1, 1) + grid, g["u"]),
                               rtol=1e-14)


def test_gelu_against_normal_table():
    g = _load("normal_cdf_table.json")
    z = np.array(g["z"])
    np.testing.assert_allclose(O.gelu(z), z * np.array(g["Phi"]), rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------------
# closed forms of single-mode inputs
# --------------------------------------------------------------------------

def _theta(grid, k):
    mesh = np.meshgrid(*[np.arange(n) for n in grid], indexing="ij")
    return 2 * np.pi * sum(kj * m / n for kj, m, n in zip(k, mesh, grid))


@pytest.mark.parametrize("grid,modes,kstar", [
    ((16, 12), (4, 5), (3, 2)),        # positive non-last wavenumber
    ((16, 12), (4, 5), (14, 4)),       # negative non-last wavenumber (-2)
    ((8, 6, 10), (2, 2, 3), (7, 1, 2)),
    ((20,), (6,), (5,)),
])
def test_single_mode_cosine_and_sine(grid, modes, kstar):
    """x = cos(theta(k*)) gives |R| cos(theta + arg R); sin gives |R| sin(theta + arg R)."""
    rng = np.random.default_rng(5)
    ci, co = 3, 2
    n_k = O.num_modes(grid, modes)
    r = _rand_r(rng, ci, co, n_k)
    kept = np.array(np.meshgrid(*[O.axis_wavenumbers(n, m, j == len(grid) - 1)
                                  for j, (n, m) in enumerate(zip(grid, modes))],
                                indexing="ij")).reshape(len(grid), -1).T
    kidx = int(np.nonzero((kept == np.array(kstar)).all(axis=1))[0][0])
    th = _theta(grid, kstar)
    for fn, shift in ((np.cos, 0.0), (np.sin, -np.pi / 2)):
        x = np.zeros((1, ci) + grid)
        x[0, 1] = fn(th)
        y, _ = O.spectral_conv_fwd(x, r, modes)
        rr = r[1, :, kidx]
        expect = np.abs(rr)[:, None] * np.cos(th.ravel()[None, :] + np.angle(rr)[:, None] + shift)
        np.testing.assert_allclose(y.reshape(co, -1), expect, atol=1e-12)


def test_single_mode_dc_column_two_term_closed_form():
    """k*_last = 0, k*_0 != 0: both +-k*_0 are kept, each with its own weight, c = 1."""
    grid, modes = (12, 10), (3, 4)
    rng = np.random.default_rng(6)
    n_k = O.num_modes(grid, modes)
    r = _rand_r(rng, 1, 1, n_k)
    k0 = 2
    th = _theta(grid, (k0, 0))
    x = np.cos(th)[None, None]
    y, _ = O.spectral_conv_fwd(x, r, modes)
    m_last = modes[1]
    r_pos = r[0, 0, k0 * m_last + 0]
    r_neg = r[0, 0, (modes[0] + (modes[0] - k0)) * m_last + 0]   # row N0 - k0 = 10
    expect = 0.5 * np.real(r_pos * np.exp(1j * th) + r_neg * np.exp(-1j * th))
    np.testing.assert_allclose(y[0, 0], expect, atol=1e-12)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid", [(8, 6), (6, 7), (4, 6, 8), (9,), (10,)])
def test_identity_weights_all_modes_reproduce_input(grid):
    d = len(grid)
    modes = tuple(n // 2 for n in grid[:-1]) + (grid[-1] // 2 + 1,)
    if any(2 * m != n for m, n in zip(modes[:-1], grid[:-1])):
        pytest.skip("odd non-last axis cannot be split into +- blocks covering it")
    c = 3
    n_k = O.num_modes(grid, modes)
    r = np.zeros((c, c, n_k), complex)
    for i in range(c):
        r[i, i, :] = 1.0
    x = np.random.default_rng(1).standard_normal((2, c) + grid)
    y, _ = O.spectral_conv_fwd(x, r, modes)
    np.testing.assert_allclose(y, x, atol=1e-12)


@pytest.mark.parametrize("grid", [(8, 6), (4, 6, 8), (10,), (4, 9)])
def test_parseval_full_half_spectrum(grid):
    modes = tuple(n // 2 for n in grid[:-1]) + (grid[-1] // 2 + 1,)
    x = np.random.default_rng(2).standard_normal((2, 3) + grid)
    xhat = O.truncated_dft(x, modes)
    c = O.mode_weights(grid, modes)
    lhs = (x ** 2).reshape(2, 3, -1).sum(-1)
    rhs = (c * np.abs(xhat) ** 2).sum(-1) / np.prod(grid)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12)


def test_linearity_in_x_and_r():
    grid, modes = (12, 10), (3, 4)
    rng = np.random.default_rng(3)
    x1, x2 = rng.standard_normal((2, 2, 3) + grid)
    n_k = O.num_modes(grid, modes)
    r1, r2 = _rand_r(rng, 3, 4, n_k), _rand_r(rng, 3, 4, n_k)
    al, be = 0.7, -1.3
    y = O.spectral_conv_fwd(al * x1 + be * x2, r1, modes)[0]
    np.testing.assert_allclose(y, al * O.spectral_conv_fwd(x1, r1, modes)[0]
                               + be * O.spectral_conv_fwd(x2, r1, modes)[0], atol=1e-12)
    y = O.spectral_conv_fwd(x1, al * r1 + be * r2, modes)[0]
    np.testing.assert_allclose(y, al * O.spectral_conv_fwd(x1, r1, modes)[0]
                               + be * O.spectral_conv_fwd(x1, r2, modes)[0], atol=1e-12)


def _brute_dft(s, grid, modes):
    """Non-separable d-dimensional sum, one kept mode at a time."""
    d = len(grid)
    kept = [O.axis_wavenumbers(n, m, j == d - 1) for j, (n, m) in enumerate(zip(grid, modes))]
    ks = np.array(np.meshgrid(*kept, indexing="ij")).reshape(d, -1).T
    out = np.zeros(s.shape[:2] + (len(ks),), complex)
    for q, k in enumerate(ks):
        out[..., q] = (s * np.exp(-1j * _theta(grid, k))).reshape(s.shape[:2] + (-1,)).sum(-1)
    return out, ks


@pytest.mark.parametrize("grid,modes", [((8, 8), (3, 4)), ((6, 10), (2, 5)), ((9, 7), (4, 4)),
                                        ((4, 6, 8), (1, 2, 3)), ((7,), (3,))])
def test_brute_force_forward_and_inverse(grid, modes):
    rng = np.random.default_rng(4)
    s = rng.standard_normal((2, 3) + grid)
    ref, ks = _brute_dft(s, grid, modes)
    np.testing.assert_allclose(O.truncated_dft(s, modes), ref, atol=1e-10)
    v = rng.standard_normal(ref.shape) + 1j * rng.standard_normal(ref.shape)
    inv = np.zeros(s.shape)
    for q, k in enumerate(ks):
        inv += np.real(v[..., q][..., None].reshape(2, 3, *([1] * len(grid)))
                       * np.exp(1j * _theta(grid, k)))
    np.testing.assert_allclose(O.inverse_sum(v, grid, modes), inv, atol=1e-10)


@pytest.mark.parametrize("grid,modes", [((16, 12), (4, 5)), ((8, 6, 10), (2, 3, 4)), ((32,), (7,)),
                                        ((15, 9), (5, 5))])
def test_against_numpy_rfftn(grid, modes):
    """Library check: NumPy's rfftn, sliced to K in storage order."""
    s = np.random.default_rng(7).standard_normal((2, 3) + grid)
    full = np.fft.rfftn(s, axes=tuple(range(2, 2 + len(grid))))
    idx = [O.axis_wavenumbers(n, m, j == len(grid) - 1) for j, (n, m) in enumerate(zip(grid, modes))]
    ref = full[np.ix_(range(2), range(3), *idx)].reshape(2, 3, -1)
    np.testing.assert_allclose(O.truncated_dft(s, modes), ref, atol=1e-10)


def test_inverse_against_numpy_irfftn_all_modes():
    """With all modes kept, (1/N) c_k Re(...) is NumPy's irfftn of a Hermitian spectrum."""
    grid = (8, 10)
    modes = (4, 6)
    s = np.random.default_rng(8).standard_normal((2, 3) + grid)
    full = np.fft.rfftn(s, axes=(2, 3))
    xhat = O.truncated_dft(s, modes)
    w = O.mode_weights(grid, modes) / np.prod(grid)
    np.testing.assert_allclose(O.inverse_sum(xhat * w, grid, modes),
                               np.fft.irfftn(full, s=grid, axes=(2, 3)), atol=1e-12)


@pytest.mark.parametrize("grid,modes", [((12, 10), (3, 4)), ((6, 8, 10), (2, 2, 3))])
def test_adjoint_identity(grid, modes):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, 3) + grid)
    n_k = O.num_modes(grid, modes)
    v = rng.standard_normal((2, 3, n_k)) + 1j * rng.standard_normal((2, 3, n_k))
    lhs = np.real(np.sum(np.conj(O.truncated_dft(x, modes)) * v))
    rhs = np.sum(x * O.inverse_sum(v, grid, modes))
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12)


@pytest.mark.parametrize("grid,modes", [((8, 6), (3, 3)), ((5, 4, 6), (2, 1, 2))])
def test_kept_mode_storage_order_single_modes(grid, modes):
    """Storage order of K from single-mode inputs: on a non-last axis the kept
    rows are the positive block 0..m-1 and then the negative block -m..-1
    (= N-m..N-1), row-major over the axes.  x = cos(theta(k*, n)) has the
    spectrum (N/2)(delta(k*) + delta(-k*)); with k*_last >= 1 only k* is kept,
    so exactly one stored entry is N/2 and it sits at k*'s slot."""
    d = len(grid)
    n_total = int(np.prod(grid))
    # signed wavenumbers of each axis in the documented storage order
    rows = [list(range(m)) + list(range(-m, 0)) for m in modes[:-1]] + [list(range(modes[-1]))]
    shape = tuple(len(r) for r in rows)
    idx = np.indices(grid)
    for slot in np.ndindex(*shape):
        k_signed = [rows[j][slot[j]] for j in range(d)]
        if k_signed[-1] == 0:
            continue
        phase = sum(2 * np.pi * k_signed[j] * idx[j] / grid[j] for j in range(d))
        x = np.cos(phase)[None, None]
        got = O.truncated_dft(x, modes).ravel()
        expect = np.zeros(len(got), complex)
        expect[np.ravel_multi_index(slot, shape)] = n_total / 2
        np.testing.assert_allclose(got, expect, atol=1e-9, err_msg=str(k_signed))


def test_mode_weights_odd_and_even_last_axis():
    np.testing.assert_array_equal(O.mode_weights((8,), (5,)), [1, 2, 2, 2, 1])
    np.testing.assert_array_equal(O.mode_weights((9,), (5,)), [1, 2, 2, 2, 2])
    np.testing.assert_array_equal(O.mode_weights((4, 8), (1, 3)), [1, 2, 2, 1, 2, 2])


def test_rejects_overlapping_modes():
    with pytest.raises(ValueError):
        O.axis_wavenumbers(8, 5, False)
    with pytest.raises(ValueError):
        O.axis_wavenumbers(8, 6, True)


# --------------------------------------------------------------------------
# finite differences of the backward passes
# --------------------------------------------------------------------------

H = 1e-6


def _fd_dir(f, x, dx):
    return (f(x + H * dx) - f(x - H * dx)) / (2 * H)


@pytest.mark.parametrize("flags", [0, O.TANH_PREACT])
def test_spectral_conv_bwd_finite_differences(flags):
    grid, modes = (8, 6), (2, 3)
    rng = np.random.default_rng(10)
    x = rng.standard_normal((2, 3) + grid)
    n_k = O.num_modes(grid, modes)
    r = _rand_r(rng, 3, 4, n_k)
    g = rng.standard_normal((2, 4) + grid)
    y, xhat = O.spectral_conv_fwd(x, r, modes, flags)
    dx, d_r = O.spectral_conv_bwd(x, r, xhat, g, modes, flags)
    loss_x = lambda xx: np.sum(O.spectral_conv_fwd(xx, r, modes, flags)[0] * g)
    loss_r = lambda rr: np.sum(O.spectral_conv_fwd(x, rr, modes, flags)[0] * g)
    v = rng.standard_normal(x.shape)
    np.testing.assert_allclose(_fd_dir(loss_x, x, v), np.sum(dx * v), rtol=1e-6)
    vr = rng.standard_normal(r.shape)
    np.testing.assert_allclose(_fd_dir(loss_r, r, vr), np.sum(d_r.real * vr), rtol=1e-6)
    np.testing.assert_allclose(_fd_dir(loss_r, r, 1j * vr), np.sum(d_r.imag * vr), rtol=1e-6)


@pytest.mark.parametrize("flags", [0, O.TANH_PREACT])
def test_spectral_conv_bwd_cp_finite_differences(flags):
    """Every CP factor's gradient (real and imaginary directions) and dx against
    central differences of L = <spectral_conv_fwd_cp(x, factors), g>."""
    grid, modes, rank = (8, 6), (2, 3), 3
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, 3) + grid)
    n_k = O.num_modes(grid, modes)

    def cplx(*shape):
        return rng.standard_normal(shape) + 1j * rng.standard_normal(shape)
    fac = [cplx(rank), cplx(3, rank), cplx(4, rank), cplx(n_k, rank)]
    g = rng.standard_normal((2, 4) + grid)
    _, xhat = O.spectral_conv_fwd_cp(x, *fac, modes, flags)
    dx, *dfac = O.spectral_conv_bwd_cp(x, *fac, xhat, g, modes, flags)
    loss_x = lambda xx: np.sum(O.spectral_conv_fwd_cp(xx, *fac, modes, flags)[0] * g)
    v = rng.standard_normal(x.shape)
    np.testing.assert_allclose(_fd_dir(loss_x, x, v), np.sum(dx * v), rtol=1e-6)
    for j in range(4):
        def loss_j(z, j=j):
            f2 = list(fac)
            f2[j] = z
            return np.sum(O.spectral_conv_fwd_cp(x, *f2, modes, flags)[0] * g)
        vj = rng.standard_normal(fac[j].shape)
        np.testing.assert_allclose(_fd_dir(loss_j, fac[j], vj), np.sum(dfac[j].real * vj),
                                   rtol=1e-5, atol=1e-9)
        np.testing.assert_allclose(_fd_dir(loss_j, fac[j], 1j * vj), np.sum(dfac[j].imag * vj),
                                   rtol=1e-5, atol=1e-9)


def test_cp_factor_grads_of_a_rank_one_weight_by_hand():
    """Rank 1 with unit factors: R = lam a b c everywhere, so each factor's
    gradient is the sum of dR times the conjugate of the other three."""
    d_r = np.arange(2 * 3 * 4).reshape(2, 3, 4) * (1 + 0.5j)
    lam, a, b, c = np.array([2.0]), np.ones((2, 1)), np.ones((3, 1)) * 1j, np.ones((4, 1))
    dlam, da, db, dc = O.cp_factor_grads(d_r, lam, a, b, c)
    total = d_r.sum()
    assert np.allclose(dlam, [total * (-1j)])             # conj(a b c) = -i
    assert np.allclose(da[:, 0], d_r.sum(axis=(1, 2)) * 2 * (-1j))
    assert np.allclose(db[:, 0], d_r.sum(axis=(0, 2)) * 2)
    assert np.allclose(dc[:, 0], d_r.sum(axis=(0, 1)) * 2 * (-1j))


@pytest.mark.parametrize("grid,modes,flags", [((8, 6), (2, 3), 0), ((8, 6), (2, 3), O.TANH_PREACT),
                                              ((4, 6, 5), (1, 2, 3), 0), ((10,), (4,), O.NO_ACT)])
def test_block_bwd_finite_differences(grid, modes, flags):
    rng = np.random.default_rng(11)
    ci, co = 3, 4
    x = rng.standard_normal((2, ci) + grid)
    n_k = O.num_modes(grid, modes)
    r = _rand_r(rng, ci, co, n_k) * 0.1
    w = rng.standard_normal((co, ci))
    b = rng.standard_normal(co)
    g = rng.standard_normal((2, co) + grid)
    y, pre, xhat = O.block_fwd(x, r, w, b, modes, flags)
    dx, d_r, d_w, d_b = O.block_bwd(x, r, w, pre, xhat, g, modes, flags)

    def loss(xx=x, rr=r, ww=w, bb=b):
        return np.sum(O.block_fwd(xx, rr, ww, bb, modes, flags)[0] * g)

    v = rng.standard_normal(x.shape)
    np.testing.assert_allclose(_fd_dir(lambda t: loss(xx=t), x, v), np.sum(dx * v), rtol=1e-6)
    vr = rng.standard_normal(r.shape)
    np.testing.assert_allclose(_fd_dir(lambda t: loss(rr=t), r, vr), np.sum(d_r.real * vr), rtol=1e-6)
    np.testing.assert_allclose(_fd_dir(lambda t: loss(rr=t), r, 1j * vr), np.sum(d_r.imag * vr),
                               rtol=1e-6)
    vw = rng.standard_normal(w.shape)
    np.testing.assert_allclose(_fd_dir(lambda t: loss(ww=t), w, vw), np.sum(d_w * vw), rtol=1e-6)
    vb = rng.standard_normal(b.shape)
    np.testing.assert_allclose(_fd_dir(lambda t: loss(bb=t), b, vb), np.sum(d_b * vb), rtol=1e-6)


def test_gelu_grad_finite_differences():
    p = np.linspace(-4, 4, 41)
    np.testing.assert_allclose(O.gelu_grad(p), (O.gelu(p + H) - O.gelu(p - H)) / (2 * H), atol=1e-8)


def test_network_backward_with_mse_finite_differences():
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "f32", 2, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    a, params, t = inp["a"], inp["params"], inp["target"]
    for key in ("R",):
        params[key] = [r * 20 for r in params[key]]     # make the spectral branch matter

    def loss(pp):
        return O.mse(O.forward(a, pp, modes), t)[0]

    u, saves = O.forward(a, params, modes, save=True)
    _, du = O.mse(u, t)
    grads = O.backward(a, params, saves, du, modes)
    rng = np.random.default_rng(12)
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        v = rng.standard_normal(np.shape(params[key]))
        f = lambda s: loss({**params, key: params[key] + s * v})
        np.testing.assert_allclose((f(H) - f(-H)) / (2 * H), np.sum(grads[key] * v), rtol=1e-6,
                                   err_msg=key)
    for key in ("W", "b", "R"):
        for l in range(2):
            v = rng.standard_normal(np.shape(params[key][l]))
            for unit in ((1.0, 1j) if key == "R" else (1.0,)):
                def f(s):
                    lst = list(params[key])
                    lst[l] = lst[l] + s * unit * v
                    return loss({**params, key: lst})
                fd = (f(H) - f(-H)) / (2 * H)
                gg = grads[key][l]
                an = np.sum((gg.real if unit == 1.0 else gg.imag) * v) if key == "R" \
                    else np.sum(gg * v)
                np.testing.assert_allclose(fd, an, rtol=1e-6, err_msg=f"{key}[{l}] {unit}")


def test_mse_value_and_gradient():
    u = np.array([[1.0, 2.0], [3.0, 5.0]])
    t = np.array([[1.0, 0.0], [3.0, 4.0]])
    loss, du = O.mse(u, t)
    assert loss == pytest.approx((0 + 4 + 0 + 1) / 4)
    np.testing.assert_allclose(du, [[0, 1.0], [0, 0.5]])


# --------------------------------------------------------------------------
# input generators (inputs, not results: moments and spectral slope only)
# --------------------------------------------------------------------------

def test_grf_moments_and_spectrum_slope():
    rng = np.random.default_rng(0)
    f = synth.gaussian_random_field(rng, 8, (64, 64))
    assert np.allclose(f.mean(axis=(1, 2)), 0, atol=1e-12)
    assert np.allclose(f.std(axis=(1, 2)), 1, atol=1e-12)
    p = (np.abs(np.fft.rfft2(f)) ** 2).mean(0)
    # power ratio between |k| = 2 and |k| = 8 on the first row, averaged over samples
    ratio = p[0, 2] / p[0, 8]
    expect = ((1 + 64) / (1 + 4)) ** 2
    assert 0.3 * expect < ratio < 3 * expect


def test_bf16_rounding_is_round_to_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5])
    out = synth.quantize(vals, "bf16")
    np.testing.assert_array_equal(out, [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5])


# --------------------------------------------------------------------------
# training loop: Adam, storage rounding, precision schedule
# --------------------------------------------------------------------------

def test_adam_hand_derived_two_steps():
    g = _load("adam_two_steps_hand.json")
    theta, m, v = np.array([g["theta0"]]), np.zeros(1), np.zeros(1)
    for t, grad in enumerate(g["grads"], start=1):
        theta, m, v = O.adam_update(theta, m, v, np.array([grad]), t, g["lr"], g["beta1"],
                                    g["beta2"], g["eps"])
        np.testing.assert_allclose(m, [g["m"][t - 1]], rtol=1e-14)
        np.testing.assert_allclose(v, [g["v"][t - 1]], rtol=1e-14)
        np.testing.assert_allclose(theta, [g["theta"][t - 1]], rtol=1e-14)


@pytest.mark.parametrize("grad", [3.0, -0.5, 1e-6, -2e-7])
def test_adam_constant_gradient_closed_form(grad):
    """With a constant gradient the bias-corrected moments are exactly g and g^2,
    so every step moves theta by lr g / (|g| + eps); eps matters for tiny g."""
    lr, eps, steps = 0.05, 1e-8, 7
    theta, m, v = np.array([0.3]), np.zeros(1), np.zeros(1)
    for t in range(1, steps + 1):
        theta, m, v = O.adam_update(theta, m, v, np.array([grad]), t, lr, 0.9, 0.999, eps)
    expect = 0.3 - steps * lr * grad / (abs(grad) + eps)
    np.testing.assert_allclose(theta, [expect], rtol=1e-12)


def test_adam_decoupled_weight_decay_closed_form():
    """A zero gradient leaves both moments at zero; decoupled decay alone shrinks
    theta by (1 - lr wd) per step."""
    lr, wd = 0.01, 0.5
    theta, m, v = np.array([2.0, -1.0]), np.zeros(2), np.zeros(2)
    for t in range(1, 6):
        theta, m, v = O.adam_update(theta, m, v, np.zeros(2), t, lr, weight_decay=wd)
    np.testing.assert_allclose(theta, np.array([2.0, -1.0]) * (1 - lr * wd) ** 5, rtol=1e-14)
    assert not m.any() and not v.any()


def test_adam_converges_on_a_quadratic():
    rng = np.random.default_rng(13)
    curv = rng.uniform(0.5, 5.0, 16)
    centre = rng.standard_normal(16)
    theta, m, v = np.zeros(16), np.zeros(16), np.zeros(16)
    for t in range(1, 3001):
        theta, m, v = O.adam_update(theta, m, v, curv * (theta - centre), t, 0.01)
    np.testing.assert_allclose(theta, centre, atol=1e-3)


def test_round_to_storage_ties_to_even():
    vals = [1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 1.0 + 2 ** -8 + 2 ** -20]
    np.testing.assert_array_equal(O.round_to_storage(vals, "bf16"),
                                  [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 1.0 + 2 ** -7])
    np.testing.assert_array_equal(O.round_to_storage([1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11], "f16"),
                                  [1.0, 1.0 + 2 ** -9])
    np.testing.assert_array_equal(O.round_to_storage([1.0 + 2 ** -24], "f32"), [1.0])


def test_precision_schedule_phases():
    phases = [(0, "bf16"), (4, "f32")]
    assert [O.dtype_at(phases, t) for t in range(6)] == ["bf16"] * 4 + ["f32"] * 2
    assert O.dtype_at([(0, "f16")], 1000) == "f16"
    with pytest.raises(ValueError):
        O.dtype_at([(2, "f32")], 0)


def test_train_first_step_is_adam_first_step():
    """The loop's first step moves every parameter component by lr g / (|g| + eps),
    g the network gradient at the starting point (Adam's first step in closed form)."""
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "f32", 2, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    a, params, t = inp["a"], inp["params"], inp["target"]
    lr, eps = 1e-2, 1e-8
    new, losses = O.train(a, t, params, modes, [(0, "f32")], 1, lr, eps=eps)
    q = {k: ([O.round_to_storage(x.real, "f32") + 1j * O.round_to_storage(x.imag, "f32")
              if np.iscomplexobj(x) else O.round_to_storage(x, "f32") for x in v]
             if isinstance(v, list) else O.round_to_storage(v, "f32")) for k, v in params.items()}
    a_q, t_q = O.round_to_storage(a, "f32"), O.round_to_storage(t, "f32")
    u, saves = O.forward(a_q, q, modes, save=True)
    loss, du = O.mse(u, t_q)
    assert losses == [loss]
    grads = O.backward(a_q, q, saves, du, modes)

    def step(g):
        return lr * g / (np.abs(g) + eps)

    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        np.testing.assert_allclose(new[key], params[key] - step(grads[key]), rtol=1e-12, atol=1e-15)
    for l in range(2):
        np.testing.assert_allclose(new["W"][l], params["W"][l] - step(grads["W"][l]), rtol=1e-12)
        r = params["R"][l]
        expect = (r.real - step(grads["R"][l].real)) + 1j * (r.imag - step(grads["R"][l].imag))
        np.testing.assert_allclose(new["R"][l], expect, rtol=1e-12)


def test_train_loss_decreases_across_a_precision_switch():
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "bf16", 2, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    _, losses = O.train(inp["a"], inp["target"], inp["params"], modes, [(0, "bf16"), (3, "f32")],
                        6, 1e-2)
    assert all(b < a for a, b in zip(losses, losses[1:]))
