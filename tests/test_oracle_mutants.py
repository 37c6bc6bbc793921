"""Planted mistakes in the CPU oracle: each must make a pin fail (test_oracle.py,
test_contraction.py).

Every mutant below is a plausible slip in one step of the oracle: a sign, a
conjugation, a normalisation, a mode weight, a mode order, a dropped term or a
transposed operand. For each mutant the test runs the oracle's pin suite in a
child process with the mutant patched in (into ``oracle.fno_oracle``, where
the oracle's own functions look names up, and into the ``oracle`` package) and
requires that the suite fails on an assertion. The unmutated suite must pass
under the same harness. Mutations live only here, on the CPU; nothing else
imports this file.

    python tests/test_oracle_mutants.py <mutant>    # run the pins under one mutant
"""

import math
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = [os.path.join(ROOT, "tests", "test_oracle.py"),
        os.path.join(ROOT, "tests", "test_contraction.py")]


def _mutants(fo):
    """name -> {attribute of oracle.fno_oracle: replacement}."""
    orig_dft, orig_inv = fo.truncated_dft, fo.inverse_sum
    orig_weights, orig_axis = fo.mode_weights, fo.axis_wavenumbers

    def dft_sign(s, modes):                     # forward transform with exp(+i theta)
        return np.conj(orig_dft(np.asarray(s, np.float64), modes))

    def inverse_sign(v, grid, modes):           # inverse with exp(-i theta)
        return orig_inv(np.conj(np.asarray(v, np.complex128)), grid, modes)

    def weights_times_n(grid, modes):           # 1/N of the inverse forgotten
        return orig_weights(grid, modes) * float(np.prod(grid))

    def weights_all_two(grid, modes):           # DC / Nyquist columns weighted 2
        return np.full_like(orig_weights(grid, modes), 2.0)

    def weights_all_one(grid, modes):           # conjugate half never doubled
        return np.ones_like(orig_weights(grid, modes))

    def weights_dc_only(grid, modes):           # Nyquist column weighted 2
        w = orig_weights(grid, modes)
        kl = orig_axis(grid[-1], modes[-1], True)
        c_last = np.where(kl == 0, 1.0, 2.0)
        return np.tile(c_last, w.size // c_last.size)

    def axis_reversed_negative(n_points, m, last):   # negative block stored N-1 .. N-m
        if last:
            return orig_axis(n_points, m, last)
        if not 1 <= 2 * m <= n_points:
            raise ValueError("non-last-axis modes out of range")
        return np.concatenate([np.arange(m), np.arange(n_points - 1, n_points - m - 1, -1)])

    def spectral_fwd_conj_r(x, r, modes, flags=0):   # mixing with conj(R)
        x = np.asarray(x, np.float64)
        grid = x.shape[2:]
        s = np.tanh(x) if flags & fo.TANH_PREACT else x
        xhat = fo.truncated_dft(s, modes)
        yhat = np.einsum("bik,iok->bok", xhat, np.conj(np.asarray(r, np.complex128)))
        w = fo.mode_weights(grid, modes) / float(np.prod(grid))
        return fo.inverse_sum(yhat * w, grid, modes), xhat

    def spectral_fwd_tanh_skipped(x, r, modes, flags=0):   # tanh flag ignored
        return _spectral_fwd_ref(fo, x, r, modes, 0)

    def gelu_tanh_approx(p):                    # tanh approximation instead of erf
        p = np.asarray(p, np.float64)
        return 0.5 * p * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (p + 0.044715 * p ** 3)))

    def gelu_grad_cdf_only(p):                  # p * phi(p) term dropped
        p = np.asarray(p, np.float64)
        return 0.5 * (1.0 + np.vectorize(math.erf)(p / math.sqrt(2.0)))

    def spectral_bwd(variant):
        def f(x, r, xhat, dy, modes, flags=0):
            x = np.asarray(x, np.float64)
            grid = x.shape[2:]
            r = np.asarray(r, np.complex128)
            w = fo.mode_weights(grid, modes) / float(np.prod(grid))
            if variant == "dyhat_unweighted":    # c_k / N left out of the cotangent
                w = np.ones_like(w)
            dyhat = fo.truncated_dft(np.asarray(dy, np.float64), modes) * w
            xh = xhat if variant == "dr_no_conj" else np.conj(xhat)
            d_r = np.einsum("bik,bok->iok", xh, dyhat)
            rr = r if variant == "dxhat_no_conj" else np.conj(r)
            dxhat = np.einsum("bok,iok->bik", dyhat, rr)
            ds = fo.inverse_sum(dxhat, grid, modes)
            if flags & fo.TANH_PREACT and variant != "tanh_grad_missing":
                ds = ds * (1.0 - np.tanh(x) ** 2)
            return ds, d_r
        return f

    def block_bwd(variant):
        def f(x, r, w, pre, xhat, dy, modes, flags=0):
            x = np.asarray(x, np.float64)
            dy = np.asarray(dy, np.float64)
            dz = dy if flags & fo.NO_ACT else dy * fo.gelu_grad(pre)
            spatial = tuple(range(2, x.ndim))
            db = dz.sum(axis=(0,) + spatial)
            if variant == "db_dropped":
                db = np.zeros_like(db)
            d_w = fo._outer_sum(dz, x)
            dx_spec, d_r = fo.spectral_conv_bwd(x, r, xhat, dz, modes, flags)
            skip = np.zeros_like(x) if variant == "skip_grad_dropped" else \
                fo._pointwise(np.asarray(w, np.float64).T, dz)
            return skip + dx_spec, d_r, d_w, db
        return f

    fo_backward = fo.backward

    def backward_q2_from_h(a, params, saves, du, modes, flags=0):   # dQ2 uses pre-GELU h
        g = fo_backward(a, params, saves, du, modes, flags)
        g["Q2"] = fo._outer_sum(np.asarray(du, np.float64), saves["h"])
        return g

    def lift_bias_dropped(a, p_mat, p_vec):
        a = np.asarray(a, np.float64)
        return fo._pointwise(p_mat, a)

    def mse_half_gradient(u, target):            # factor 2 of d(mean sq)/du dropped
        diff = np.asarray(u, np.float64) - np.asarray(target, np.float64)
        return float(np.mean(diff * diff)), diff / diff.size

    def adam(variant):
        def f(theta, m, v, g, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
            theta = np.asarray(theta, np.float64)
            g = np.asarray(g, np.float64)
            if variant == "coupled_decay":       # L2 term folded into the gradient
                g = g + weight_decay * theta
            m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
            v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
            if variant == "no_bias_correction":
                m_hat, v_hat = m, v
            else:
                m_hat, v_hat = m / (1.0 - beta1 ** t), v / (1.0 - beta2 ** t)
            if variant == "eps_inside_sqrt":
                denom = np.sqrt(v_hat + eps)
            else:
                denom = np.sqrt(v_hat) + eps
            decay = 0.0 if variant == "coupled_decay" else lr * weight_decay * theta
            return theta - lr * m_hat / denom - decay, m, v
        return f

    def bf16_truncating(x, dtype):              # bf16 rounding by truncation
        if dtype != "bf16":
            return orig_round(x, dtype)
        bits = np.asarray(x, np.float64).astype(np.float32).view(np.uint32)
        return (bits & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)

    orig_round = fo.round_to_storage

    def dtype_at_late(phases, step):            # a phase starts one step late
        current = None
        for start, dtype in phases:
            if start < step or start == 0:
                current = dtype
        if current is None:
            raise ValueError("no phase covers step %d" % step)
        return current

    def cp_factor_conjugated(lam, a, b, c):     # conj(c) in the CP weight
        return np.einsum("r,ir,or,kr->iok", np.asarray(lam, np.complex128),
                         np.asarray(a, np.complex128), np.asarray(b, np.complex128),
                         np.conj(np.asarray(c, np.complex128)))

    def cp_lambda_dropped(lam, a, b, c):        # CP weights without lam
        return np.einsum("ir,or,kr->iok", np.asarray(a, np.complex128),
                         np.asarray(b, np.complex128), np.asarray(c, np.complex128))

    def cp_grads_unconjugated(d_r, lam, a, b, c):   # factor gradients without conj
        d_r = np.asarray(d_r, np.complex128)
        lam, a, b, c = (np.asarray(v, np.complex128) for v in (lam, a, b, c))
        return (np.einsum("iok,ir,or,kr->r", d_r, a, b, c),
                np.einsum("iok,r,or,kr->ir", d_r, lam, b, c),
                np.einsum("iok,r,ir,kr->or", d_r, lam, a, c),
                np.einsum("iok,r,ir,or->kr", d_r, lam, a, b))

    def projection_without_gelu(v, q1_mat, q1_vec, q2_mat, q2_vec):   # hidden layer linear
        v = np.asarray(v, np.float64)
        d = v.ndim - 2
        h = fo._pointwise(q1_mat, v) + fo._bcast(q1_vec, d)
        return fo._pointwise(q2_mat, h) + fo._bcast(q2_vec, d)

    return {
        "projection_without_gelu": {"projection": projection_without_gelu},
        "cp_factor_conjugated": {"cp_weights": cp_factor_conjugated},
        "cp_lambda_dropped": {"cp_weights": cp_lambda_dropped},
        "cp_grads_unconjugated": {"cp_factor_grads": cp_grads_unconjugated},
        "adam_no_bias_correction": {"adam_update": adam("no_bias_correction")},
        "adam_eps_inside_sqrt": {"adam_update": adam("eps_inside_sqrt")},
        "adam_coupled_decay": {"adam_update": adam("coupled_decay")},
        "bf16_truncating": {"round_to_storage": bf16_truncating},
        "schedule_phase_late": {"dtype_at": dtype_at_late},
        "dft_sign": {"truncated_dft": dft_sign},
        "inverse_sign": {"inverse_sum": inverse_sign},
        "inverse_unscaled": {"mode_weights": weights_times_n},
        "ck_all_two": {"mode_weights": weights_all_two},
        "ck_all_one": {"mode_weights": weights_all_one},
        "ck_nyquist_doubled": {"mode_weights": weights_dc_only},
        "negative_block_reversed": {"axis_wavenumbers": axis_reversed_negative},
        "mix_conj_r": {"spectral_conv_fwd": spectral_fwd_conj_r},
        "tanh_preact_ignored": {"spectral_conv_fwd": spectral_fwd_tanh_skipped},
        "gelu_tanh_approx": {"gelu": gelu_tanh_approx},
        "gelu_grad_cdf_only": {"gelu_grad": gelu_grad_cdf_only},
        "dr_no_conj": {"spectral_conv_bwd": spectral_bwd("dr_no_conj")},
        "dxhat_no_conj": {"spectral_conv_bwd": spectral_bwd("dxhat_no_conj")},
        "dyhat_unweighted": {"spectral_conv_bwd": spectral_bwd("dyhat_unweighted")},
        "tanh_grad_missing": {"spectral_conv_bwd": spectral_bwd("tanh_grad_missing")},
        "db_dropped": {"block_bwd": block_bwd("db_dropped")},
        "skip_grad_dropped": {"block_bwd": block_bwd("skip_grad_dropped")},
        "dq2_from_preactivation": {"backward": backward_q2_from_h},
        "lift_bias_dropped": {"lift": lift_bias_dropped},
        "mse_half_gradient": {"mse": mse_half_gradient},
    }


def _spectral_fwd_ref(fo, x, r, modes, flags):
    x = np.asarray(x, np.float64)
    grid = x.shape[2:]
    s = np.tanh(x) if flags & fo.TANH_PREACT else x
    xhat = fo.truncated_dft(s, modes)
    yhat = np.einsum("bik,iok->bok", xhat, np.asarray(r, np.complex128))
    w = fo.mode_weights(grid, modes) / float(np.prod(grid))
    return fo.inverse_sum(yhat * w, grid, modes), xhat


MUTANT_NAMES = [
    "dft_sign", "inverse_sign", "inverse_unscaled", "ck_all_two", "ck_all_one",
    "ck_nyquist_doubled", "negative_block_reversed", "mix_conj_r", "tanh_preact_ignored",
    "gelu_tanh_approx", "gelu_grad_cdf_only", "dr_no_conj", "dxhat_no_conj", "dyhat_unweighted",
    "tanh_grad_missing", "db_dropped", "skip_grad_dropped", "dq2_from_preactivation",
    "lift_bias_dropped", "mse_half_gradient", "adam_no_bias_correction", "adam_eps_inside_sqrt",
    "adam_coupled_decay", "bf16_truncating", "schedule_phase_late", "cp_factor_conjugated",
    "cp_lambda_dropped", "cp_grads_unconjugated", "projection_without_gelu",
]


def _apply(name):
    sys.path.insert(0, ROOT)
    import oracle
    import oracle.fno_oracle as fo
    table = _mutants(fo)
    if name != "none":
        for attr, fn in table[name].items():
            setattr(fo, attr, fn)
            if hasattr(oracle, attr):
                setattr(oracle, attr, fn)
    return sorted(table)


def _run_pins(name):
    env = dict(os.environ)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    return subprocess.run([sys.executable, os.path.abspath(__file__), name], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_mutant_table_is_complete():
    import oracle.fno_oracle as fo
    assert sorted(_mutants(fo)) == sorted(MUTANT_NAMES)


def test_unmutated_pins_pass():
    p = _run_pins("none")
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-2000:]


@pytest.mark.parametrize("name", MUTANT_NAMES)
def test_every_planted_mistake_fails_a_pin(name):
    p = _run_pins(name)
    # pytest exit code 1: tests ran and at least one failed (not a collection error)
    assert p.returncode == 1, f"mutant {name} survived:\n" + p.stdout[-2000:] + p.stderr[-2000:]


if __name__ == "__main__":
    _apply(sys.argv[1])
    sys.exit(pytest.main(PINS + ["-q", "-x", "-p", "no:cacheprovider"]))
