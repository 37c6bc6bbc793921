"""CPU float64 oracle of the FNO spectral-convolution block and of the small FNO
network built from it.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` do.  It shares no code, tables or helpers with the CUDA
library, and it never reads a value the CUDA library produced.

Sources (web pages; cited by title and section):

* [MPFNO] "Model-Parallel Fourier Neural Operators as Learned Surrogates for
  Large-Scale Parametric PDEs" (review page), section "Proposed method": the
  network is the original FNO -- a lifting, four spectral blocks of embedding
  width 20, a projection -- and its spectral convolution is the operation
  written in FNO's linear-algebra form; gradients come from automatic
  differentiation (same section, last item).
* [MPTRAIN] "Guaranteed approximation bounds and efficient mixed-precision
  training for neural operators" (summary page), "key insights": the Fourier
  transform may run below full precision, the spectral contraction is a
  memory-bound half-precision tensor contraction, and a tanh pre-activation is
  applied before the Fourier transform.

The pages do not print the block's equations.  The oracle computes the
standard FNO block, with the readings listed below; each is repeated in the
repository's design notes.

Notation: ``x`` has shape ``[B, C, N_0, ..., N_{d-1}]``; the last axis is the
real-FFT axis.  The kept mode set ``K`` holds, on each non-last axis ``j``, the
wavenumbers ``0..m_j-1`` followed by ``N_j-m_j..N_j-1`` (positive block first,
negative block second), and on the last axis ``0..m_{d-1}-1``; ``K`` is
flattened row-major in that order.  ``theta(k, n) = 2*pi*sum_j k_j n_j / N_j``.

Readings (where the pages are silent):

1. Forward transform unnormalised, inverse scaled by ``1/N`` (``N = prod N_j``).
2. Inverse of the half spectrum: ``y[n] = (1/N) sum_{k in K} c_k Re(Y_k e^{+i theta})``
   with ``c_k = 1`` when ``k_{d-1} = 0`` or ``k_{d-1} = N_{d-1}/2`` and 2 otherwise
   (the imaginary part of a DC/Nyquist column is dropped, as a C2R inverse does).
3. GELU is the exact erf form ``p * Phi(p)``.
4. tanh pre-activation feeds the spectral branch only; the 1x1 path sees raw x.
5. Complex gradient convention: ``dZ = dL/dRe Z + i dL/dIm Z``.

Training loop (the precision-scheduling step of [MPTRAIN]): the summary page
says training may move from mixed to full precision part-way through.  It fixes
neither the optimiser nor the switch point; the readings are

6. Optimiser: Adam (Kingma and Ba, "Adam: A Method for Stochastic
   Optimization", Algorithm 1) on float32 master weights, with optional
   decoupled weight decay (Loshchilov and Hutter, "Decoupled Weight Decay
   Regularization"); the step runs on the master copy and the next forward
   reads it rounded to that step's storage dtype.
7. Schedule: a list of (first step, storage dtype) phases; by default the first
   half of the steps in half precision, then float32.

Parity pins: ``tests/test_oracle.py`` (closed forms, invariants, brute force,
library DFT, finite differences, hand-derived fixtures under ``tests/golden``).
"""

from __future__ import annotations

import math

import numpy as np

TANH_PREACT = 1
NO_ACT = 2

_SQRT1_2 = 1.0 / math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


# --------------------------------------------------------------------------
# mode bookkeeping
# --------------------------------------------------------------------------

def axis_wavenumbers(n_points: int, m: int, last: bool) -> np.ndarray:
    """Kept wavenumbers of one axis, in storage order (reading 1 of the header)."""
    if last:
        if not 1 <= m <= n_points // 2 + 1:
            raise ValueError("last-axis modes out of range")
        return np.arange(m)
    if not 1 <= 2 * m <= n_points:
        raise ValueError("non-last-axis modes out of range")
    return np.concatenate([np.arange(m), np.arange(n_points - m, n_points)])


def kept_shape(grid, modes):
    d = len(grid)
    return tuple(len(axis_wavenumbers(grid[j], modes[j], j == d - 1)) for j in range(d))


def num_modes(grid, modes) -> int:
    return int(np.prod(kept_shape(grid, modes)))


def mode_weights(grid, modes) -> np.ndarray:
    """``c_k`` over the flattened K (reading 2): 1 on the DC/Nyquist column, else 2."""
    d = len(grid)
    kl = axis_wavenumbers(grid[-1], modes[-1], True)
    nl = grid[-1]
    c_last = np.where((kl == 0) | ((nl % 2 == 0) & (kl == nl // 2)), 1.0, 2.0)
    lead = int(np.prod(kept_shape(grid, modes)[:-1])) if d > 1 else 1
    return np.tile(c_last, lead)


def _exp_matrix(n_points: int, ks: np.ndarray, sign: int) -> np.ndarray:
    """``E[k, n] = exp(sign * 2 pi i ((k n) mod N) / N)`` for the kept ``k``."""
    n = np.arange(n_points)
    phase = 2.0 * np.pi * (np.outer(ks, n) % n_points) / n_points
    return np.cos(phase) + sign * 1j * np.sin(phase)


# --------------------------------------------------------------------------
# the two truncated transforms
# --------------------------------------------------------------------------

def truncated_dft(s: np.ndarray, modes) -> np.ndarray:
    """``S[b, c, k] = sum_n s[b, c, n] exp(-i theta(k, n))`` for ``k`` in K.

    The d-dimensional sum is applied one axis at a time with explicit
    exponential matrices (the sum is separable; this only reorders it).
    Returns ``[B, C, |K|]`` complex128.
    """
    s = np.asarray(s)
    b, c = s.shape[:2]
    grid = s.shape[2:]
    d = len(grid)
    out = s.astype(np.complex128)
    for j in range(d - 1, -1, -1):
        ks = axis_wavenumbers(grid[j], modes[j], j == d - 1)
        e = _exp_matrix(grid[j], ks, -1)                       # [kept_j, N_j]
        out = np.moveaxis(np.tensordot(out, e, axes=([2 + j], [1])), -1, 2 + j)
    return out.reshape(b, c, -1)


def inverse_sum(v: np.ndarray, grid, modes) -> np.ndarray:
    """``u[b, c, n] = sum_{k in K} Re(v[b, c, k] exp(+i theta(k, n)))`` (no scale).

    ``v`` is ``[B, C, |K|]`` complex; returns ``[B, C, *grid]`` float64.
    """
    v = np.asarray(v, dtype=np.complex128)
    b, c = v.shape[:2]
    d = len(grid)
    out = v.reshape((b, c) + kept_shape(grid, modes))
    for j in range(d):
        ks = axis_wavenumbers(grid[j], modes[j], j == d - 1)
        e = _exp_matrix(grid[j], ks, +1)                       # [kept_j, N_j]
        out = np.moveaxis(np.tensordot(out, e, axes=([2 + j], [0])), -1, 2 + j)
    return out.real.copy()


# --------------------------------------------------------------------------
# activations
# --------------------------------------------------------------------------

try:  # vectorised library erf; math.erf element by element otherwise
    from scipy.special import erf as _erf
except ImportError:  # pragma: no cover
    def _erf(z):
        return np.vectorize(math.erf, otypes=[np.float64])(z)


def gelu(p: np.ndarray) -> np.ndarray:
    """Exact GELU ``p * Phi(p)``, ``Phi`` the standard normal CDF (reading 3)."""
    p = np.asarray(p, dtype=np.float64)
    return 0.5 * p * (1.0 + _erf(p * _SQRT1_2))


def gelu_grad(p: np.ndarray) -> np.ndarray:
    """``d/dp [p Phi(p)] = Phi(p) + p phi(p)``."""
    p = np.asarray(p, dtype=np.float64)
    return 0.5 * (1.0 + _erf(p * _SQRT1_2)) + p * _INV_SQRT_2PI * np.exp(-0.5 * p * p)


# --------------------------------------------------------------------------
# spectral convolution and block
# --------------------------------------------------------------------------

def _pointwise(mat: np.ndarray, v: np.ndarray) -> np.ndarray:
    """``out[b, o, n] = sum_i mat[o, i] v[b, i, n]`` (a 1x1 convolution)."""
    return np.einsum("oi,bi...->bo...", np.asarray(mat, np.float64), v)


def _outer_sum(u: np.ndarray, v: np.ndarray) -> np.ndarray:
    """``out[o, i] = sum_{b, n} u[b, o, n] v[b, i, n]`` over batch and grid points."""
    u2 = np.asarray(u, np.float64).reshape(u.shape[0], u.shape[1], -1)
    v2 = np.asarray(v, np.float64).reshape(v.shape[0], v.shape[1], -1)
    return np.einsum("bon,bin->oi", u2, v2)


def _bcast(vec: np.ndarray, d: int) -> np.ndarray:
    return np.asarray(vec, np.float64).reshape((1, -1) + (1,) * d)


def spectral_conv_fwd(x, r, modes, flags: int = 0):
    """Spectral branch of the block.

    ``s = tanh(x)`` if TANH_PREACT ([MPTRAIN] key insights) else ``x``;
    ``xhat = DFT_K(s)``; ``yhat[b,o,k] = sum_i xhat[b,i,k] r[i,o,k]``;
    ``y = (1/N) sum_k c_k Re(yhat e^{+i theta})``.
    Returns ``(y, xhat)``.
    """
    x = np.asarray(x, np.float64)
    grid = x.shape[2:]
    s = np.tanh(x) if flags & TANH_PREACT else x
    xhat = truncated_dft(s, modes)
    yhat = np.einsum("bik,iok->bok", xhat, np.asarray(r, np.complex128))
    w = mode_weights(grid, modes) / float(np.prod(grid))
    return inverse_sum(yhat * w, grid, modes), xhat


def spectral_conv_bwd(x, r, xhat, dy, modes, flags: int = 0):
    """Adjoint of :func:`spectral_conv_fwd` (gradients by differentiation, [MPFNO]).

    ``dyhat = (c_k/N) DFT_K(dy)``; ``dR = sum_b conj(xhat) dyhat``;
    ``dxhat = sum_o dyhat conj(R)``; ``ds = sum_k Re(dxhat e^{+i theta})``;
    ``dx = ds (1 - tanh^2 x)`` under TANH_PREACT, else ``ds``.
    Returns ``(dx, dR)``.
    """
    x = np.asarray(x, np.float64)
    grid = x.shape[2:]
    r = np.asarray(r, np.complex128)
    w = mode_weights(grid, modes) / float(np.prod(grid))
    dyhat = truncated_dft(np.asarray(dy, np.float64), modes) * w
    d_r = np.einsum("bik,bok->iok", np.conj(xhat), dyhat)
    dxhat = np.einsum("bok,iok->bik", dyhat, np.conj(r))
    ds = inverse_sum(dxhat, grid, modes)
    if flags & TANH_PREACT:
        ds = ds * (1.0 - np.tanh(x) ** 2)
    return ds, d_r


def block_fwd(x, r, w, bias, modes, flags: int = 0):
    """``pre = spectral(x) + W x + b``; ``y = GELU(pre)`` unless NO_ACT.

    Returns ``(y, pre, xhat)``.
    """
    x = np.asarray(x, np.float64)
    d = x.ndim - 2
    y_spec, xhat = spectral_conv_fwd(x, r, modes, flags)
    pre = y_spec + _pointwise(w, x) + _bcast(bias, d)
    y = pre if flags & NO_ACT else gelu(pre)
    return y, pre, xhat


def block_bwd(x, r, w, pre, xhat, dy, modes, flags: int = 0):
    """Adjoint of :func:`block_fwd`: returns ``(dx, dR, dW, db)``.

    ``dz = dy * GELU'(pre)``; ``db = sum dz``; ``dW = sum dz x^T``;
    ``dx = W^T dz + spectral_bwd(dz)``.
    """
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    dz = dy if flags & NO_ACT else dy * gelu_grad(pre)
    spatial = tuple(range(2, x.ndim))
    db = dz.sum(axis=(0,) + spatial)
    d_w = _outer_sum(dz, x)
    dx_spec, d_r = spectral_conv_bwd(x, r, xhat, dz, modes, flags)
    dx = _pointwise(np.asarray(w, np.float64).T, dz) + dx_spec
    return dx, d_r, d_w, db


# --------------------------------------------------------------------------
# network: lift -> L blocks -> projection ([MPFNO] "original FNO architecture")
# --------------------------------------------------------------------------

def lift(a, p_mat, p_vec):
    """Lifting ``v_0 = P a + p`` (pointwise over the grid)."""
    a = np.asarray(a, np.float64)
    return _pointwise(p_mat, a) + _bcast(p_vec, a.ndim - 2)


def projection(v, q1_mat, q1_vec, q2_mat, q2_vec):
    """Projection ``u = Q2 GELU(Q1 v + q1) + q2`` (pointwise over the grid)."""
    v = np.asarray(v, np.float64)
    d = v.ndim - 2
    h = _pointwise(q1_mat, v) + _bcast(q1_vec, d)
    return _pointwise(q2_mat, gelu(h)) + _bcast(q2_vec, d)


def forward(a, params, modes, flags: int = 0, save: bool = False):
    """``v_0 = P a + p``; ``v_{l+1} = block_l(v_l)``; ``u = Q2 GELU(Q1 v_L + q1) + q2``.

    ``params`` is a dict with ``P, p, R (list), W (list), b (list), Q1, q1, Q2, q2``.
    Returns ``u`` or ``(u, saves)`` with the per-layer block inputs, pre-activations,
    spectra and the projection's hidden pre-activation.
    """
    a = np.asarray(a, np.float64)
    d = a.ndim - 2
    v = lift(a, params["P"], params["p"])
    xs, pres, xhats = [], [], []
    for r, w, bias in zip(params["R"], params["W"], params["b"]):
        xs.append(v)
        v, pre, xhat = block_fwd(v, r, w, bias, modes, flags)
        pres.append(pre)
        xhats.append(xhat)
    h = _pointwise(params["Q1"], v) + _bcast(params["q1"], d)
    u = projection(v, params["Q1"], params["q1"], params["Q2"], params["q2"])
    if not save:
        return u
    return u, {"x": xs, "pre": pres, "xhat": xhats, "v_last": v, "h": h}


def backward(a, params, saves, du, modes, flags: int = 0):
    """Adjoint of :func:`forward`: gradients of every parameter (and of ``a``)."""
    a = np.asarray(a, np.float64)
    du = np.asarray(du, np.float64)
    spatial = tuple(range(2, a.ndim))
    h, v = saves["h"], saves["v_last"]
    g = gelu(h)
    grads = {
        "Q2": _outer_sum(du, g),
        "q2": du.sum(axis=(0,) + spatial),
    }
    dh = _pointwise(np.asarray(params["Q2"], np.float64).T, du) * gelu_grad(h)
    grads["Q1"] = _outer_sum(dh, v)
    grads["q1"] = dh.sum(axis=(0,) + spatial)
    dv = _pointwise(np.asarray(params["Q1"], np.float64).T, dh)
    n_layers = len(params["R"])
    d_r, d_w, d_b = [None] * n_layers, [None] * n_layers, [None] * n_layers
    for l in range(n_layers - 1, -1, -1):
        dv, d_r[l], d_w[l], d_b[l] = block_bwd(
            saves["x"][l], params["R"][l], params["W"][l], saves["pre"][l],
            saves["xhat"][l], dv, modes, flags)
    grads["R"], grads["W"], grads["b"] = d_r, d_w, d_b
    grads["P"] = _outer_sum(dv, a)
    grads["p"] = dv.sum(axis=(0,) + spatial)
    grads["a"] = _pointwise(np.asarray(params["P"], np.float64).T, dv)
    return grads


def mse(u, target):
    """``L = mean((u - t)^2)`` over every element and ``dL/du = 2 (u - t) / numel``."""
    diff = np.asarray(u, np.float64) - np.asarray(target, np.float64)
    return float(np.mean(diff * diff)), 2.0 * diff / diff.size


# --------------------------------------------------------------------------
# training loop with a precision schedule (readings 6 and 7)
# --------------------------------------------------------------------------

def round_to_storage(x, dtype: str) -> np.ndarray:
    """Round to the storage dtype (round to nearest, ties to even); float64 out."""
    x = np.asarray(x, np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        bits = x.astype(np.float32).view(np.uint32).astype(np.uint64)
        keep = bits >> 16                      # the upper 16 bits survive
        rest = bits & 0xFFFF                   # the dropped half
        up = (rest > 0x8000) | ((rest == 0x8000) & (keep & 1 == 1))
        keep = keep + up.astype(np.uint64)
        return ((keep << 16) & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def adam_update(theta, m, v, g, t: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                eps: float = 1e-8, weight_decay: float = 0.0):
    """One Adam step at step number ``t`` (1-based), reading 6.

    ``m = b1 m + (1 - b1) g``; ``v = b2 v + (1 - b2) g^2``;
    ``theta -= lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps) + lr wd theta``.
    Returns ``(theta, m, v)``.
    """
    theta = np.asarray(theta, np.float64)
    g = np.asarray(g, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    theta = theta - lr * m_hat / (np.sqrt(v_hat) + eps) - lr * weight_decay * theta
    return theta, m, v


def dtype_at(phases, step: int) -> str:
    """Storage dtype of ``step`` under ``phases`` = [(first step, dtype), ...] (reading 7)."""
    current = None
    for start, dtype in phases:
        if start <= step:
            current = dtype
    if current is None:
        raise ValueError("no phase covers step %d" % step)
    return current


_PARAM_KEYS = ("P", "p", "Q1", "q1", "Q2", "q2")
_LAYER_KEYS = ("R", "W", "b")


def _map_params(fn, *trees):
    out = {}
    for key in _PARAM_KEYS:
        out[key] = fn(*[t[key] for t in trees])
    for key in _LAYER_KEYS:
        out[key] = [fn(*xs) for xs in zip(*[t[key] for t in trees])]
    return out


def _round_param(x, dtype):
    x = np.asarray(x)
    if np.iscomplexobj(x):
        return round_to_storage(x.real, dtype) + 1j * round_to_storage(x.imag, dtype)
    return round_to_storage(x, dtype)


def train(a, target, params, modes, phases, steps: int, lr: float, beta1: float = 0.9,
          beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0, flags: int = 0):
    """``steps`` Adam steps of the network on one batch under a precision schedule.

    Step ``t`` (0-based) reads the master parameters and the inputs rounded to
    ``dtype_at(phases, t)``, takes the MSE gradient of :func:`forward` there and
    applies :func:`adam_update` (step number ``t + 1``) to the float64 master
    copy.  Complex weights are updated as (re, im) pairs.  Returns
    ``(master params, losses)``.
    """
    master = _map_params(lambda x: np.array(x, dtype=np.complex128 if np.iscomplexobj(x)
                                            else np.float64), params)
    mom = _map_params(np.zeros_like, master)      # complex weights: (re, im) moments
    vel = _map_params(np.zeros_like, master)
    losses = []
    for t in range(steps):
        dt = dtype_at(phases, t)
        q = _map_params(lambda x: _round_param(x, dt), master)
        a_q, t_q = round_to_storage(a, dt), round_to_storage(target, dt)
        u, saves = forward(a_q, q, modes, flags, save=True)
        loss, du = mse(u, t_q)
        losses.append(loss)
        grads = backward(a_q, q, saves, du, modes, flags)

        def upd(th, mm, vv, gg, step=t + 1):
            if np.iscomplexobj(th):   # real and imaginary parts are separate parameters
                re = adam_update(th.real, mm.real, vv.real, np.real(gg), step, lr, beta1, beta2,
                                 eps, weight_decay)
                im = adam_update(th.imag, mm.imag, vv.imag, np.imag(gg), step, lr, beta1, beta2,
                                 eps, weight_decay)
                return re[0] + 1j * im[0], re[1] + 1j * im[1], re[2] + 1j * im[2]
            return adam_update(th, mm, vv, gg, step, lr, beta1, beta2, eps, weight_decay)

        new = {}
        for key in _PARAM_KEYS:
            new[key] = upd(master[key], mom[key], vel[key], grads[key])
        for key in _LAYER_KEYS:
            new[key] = [upd(*xs) for xs in zip(master[key], mom[key], vel[key], grads[key])]
        master = {k: ([x[0] for x in v] if isinstance(v, list) else v[0]) for k, v in new.items()}
        mom = {k: ([x[1] for x in v] if isinstance(v, list) else v[1]) for k, v in new.items()}
        vel = {k: ([x[2] for x in v] if isinstance(v, list) else v[2]) for k, v in new.items()}
    return master, losses


# --------------------------------------------------------------------------
# factorised spectral weights (TFNO, [MPTRAIN] summary; CP reading)
# --------------------------------------------------------------------------

def cp_weights(lam, a, b, c) -> np.ndarray:
    """``R[i, o, k] = sum_r lam[r] a[i, r] b[o, r] c[k, r]``: a rank-r CP weight.

    The summary page names TFNO (factorised spectral weights) without the
    factorisation; the canonical polyadic form is the reading.  Complex factors
    allowed.  Returns ``[Ci, Co, |K|]`` complex128.
    """
    return np.einsum("r,ir,or,kr->iok", np.asarray(lam, np.complex128),
                     np.asarray(a, np.complex128), np.asarray(b, np.complex128),
                     np.asarray(c, np.complex128))


def spectral_conv_fwd_cp(x, lam, a, b, c, modes, flags: int = 0):
    """:func:`spectral_conv_fwd` with the CP weight :func:`cp_weights` (definition)."""
    return spectral_conv_fwd(x, cp_weights(lam, a, b, c), modes, flags)


def cp_factor_grads(d_r, lam, a, b, c):
    """Gradients of the CP factors from the dense weight's gradient ``d_r``.

    The weight ``R[i,o,k] = sum_r lam[r] a[i,r] b[o,r] c[k,r]`` is holomorphic in
    each factor, so with the convention ``dz = dL/dRe z + i dL/dIm z`` the chain
    rule gives ``dz = sum dR conj(dR/dz)``:
    ``dlam[r] = sum_{iok} dR conj(a b c)``, ``da[i,r] = sum_{ok} dR conj(lam b c)``,
    ``db[o,r] = sum_{ik} dR conj(lam a c)``, ``dc[k,r] = sum_{io} dR conj(lam a b)``.
    Returns ``(dlam, da, db, dc)`` complex128.
    """
    d_r = np.asarray(d_r, np.complex128)
    lam, a, b, c = (np.asarray(v, np.complex128) for v in (lam, a, b, c))
    dlam = np.einsum("iok,ir,or,kr->r", d_r, np.conj(a), np.conj(b), np.conj(c))
    da = np.einsum("iok,r,or,kr->ir", d_r, np.conj(lam), np.conj(b), np.conj(c))
    db = np.einsum("iok,r,ir,kr->or", d_r, np.conj(lam), np.conj(a), np.conj(c))
    dc = np.einsum("iok,r,ir,or->kr", d_r, np.conj(lam), np.conj(a), np.conj(b))
    return dlam, da, db, dc


def spectral_conv_bwd_cp(x, lam, a, b, c, xhat, dy, modes, flags: int = 0):
    """Adjoint of :func:`spectral_conv_fwd_cp`: :func:`spectral_conv_bwd` on the
    reconstructed weight, then :func:`cp_factor_grads`.
    Returns ``(dx, dlam, da, db, dc)``."""
    dx, d_r = spectral_conv_bwd(x, cp_weights(lam, a, b, c), xhat, dy, modes, flags)
    return (dx,) + cp_factor_grads(d_r, lam, a, b, c)
