"""Training loop on the GPU against the oracle: the fused Adam + copy kernel
element by element, and the precision-scheduled trainer step by step."""

import numpy as np
import pytest

import oracle as O
from fno_testlib import rel_l2
from fourier_neural_spectral_fno_b200 import capi, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [1, 7, 4099, (1 << 20) + 3])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_adam_step_matches_oracle(n, dtype):
    """Three Adam steps from a zero state (random gradients), kernel vs oracle.

    Tolerances from float32 arithmetic: a moment is a two-term sum, so its
    error is a few units in the last place of the larger term (2^-21 of the
    largest |g|); theta moves by at most a few lr per step, each step exact to
    a few ulps of theta plus 1e-6 of the step (the betas are float32 in the
    kernel and exact in the oracle)."""
    import torch
    from fourier_neural_spectral_fno_b200.train import torch_dtype
    rng = np.random.default_rng(21)
    theta = rng.standard_normal(n).astype(np.float32)
    lr, b1, b2, eps, wd, scale = 3e-3, 0.9, 0.99, 1e-6, 0.01, 0.5
    t_d = torch.from_numpy(theta).cuda()
    m_d, v_d = torch.zeros_like(t_d), torch.zeros_like(t_d)
    out = torch.empty(n, dtype=torch_dtype(dtype), device="cuda")
    th_ref, m_ref, v_ref = theta.astype(np.float64), np.zeros(n), np.zeros(n)
    gmax = 0.0
    for step in (1, 2, 3):
        g = (rng.standard_normal(n) * np.exp(rng.uniform(-3, 1, n))).astype(np.float32)
        gmax = max(gmax, float(np.abs(g).max()) * scale)
        capi.fno_adam_step(t_d, m_d, v_d, torch.from_numpy(g).cuda(), out, step, lr, b1, b2, eps,
                           wd, scale)
        th_ref, m_ref, v_ref = O.adam_update(th_ref, m_ref, v_ref, g.astype(np.float64) * scale,
                                             step, lr, b1, b2, eps, wd)
    torch.cuda.synchronize()
    np.testing.assert_allclose(m_d.cpu().numpy(), m_ref, rtol=1e-5, atol=2.0 ** -21 * gmax)
    np.testing.assert_allclose(v_d.cpu().numpy(), v_ref, rtol=1e-5, atol=2.0 ** -21 * gmax ** 2)
    th_gpu = t_d.cpu().numpy()
    np.testing.assert_allclose(th_gpu, th_ref, rtol=2.0 ** -20, atol=3 * 1e-5 * lr)
    assert np.abs(th_gpu - theta).max() <= 3 * 4 * lr      # each step moves at most a few lr
    # the copy is the float32 master rounded to the storage dtype (same precision on both sides)
    np.testing.assert_array_equal(out.float().cpu().numpy().astype(np.float64),
                                  O.round_to_storage(th_gpu, dtype))
    # copy only: theta, m, v untouched
    before, m_before = t_d.clone(), m_d.clone()
    out2 = torch.empty_like(out)
    capi.fno_adam_step(t_d, None, None, None, out2, 1, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(t_d, before) and torch.equal(m_d, m_before)
    assert torch.equal(out2, out)


def _network(dtype, grid=(16, 12), modes=(4, 5)):
    wl = synth.Workload("tiny", "network", dtype, 2, grid, modes, 6, in_ch=3, hidden=9,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    p = inp["params"]
    p["R"] = [synth.quantize_complex(r * 6 * 6 / np.sqrt(6), dtype) for r in p["R"]]
    return wl, inp


def _flat(params):
    parts = []
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        parts.append(np.ravel(params[key]))
    for key in ("R", "W", "b"):
        for x in params[key]:
            x = np.asarray(x)
            parts.append(np.ravel(np.stack([x.real, x.imag], -1) if np.iscomplexobj(x) else x))
    return np.concatenate(parts)


def _run_trainer(wl, inp, phases, steps, lr):
    import torch
    from fourier_neural_spectral_fno_b200.train import PrecisionSchedule, Trainer
    tr = Trainer(wl.grid, wl.modes, wl.in_ch, wl.width, inp["params"],
                 PrecisionSchedule(phases), hidden=wl.hidden, n_layers=wl.n_layers, lr=lr)
    a = torch.from_numpy(np.asarray(inp["a"], np.float32)).cuda()
    t = torch.from_numpy(np.asarray(inp["target"], np.float32)).cuda()
    losses, dtypes = [], []
    for _ in range(steps):
        dtypes.append(tr.dtype if tr.dtype else phases[0][1])
        losses.append(float(tr.step(a, t).item()))
    return tr, losses, dtypes


@pytest.mark.parametrize("grid,modes", [((16, 12), (4, 5)), ((128, 64), (8, 8))])
def test_trainer_f32_matches_oracle(grid, modes):
    wl, inp = _network("f32", grid, modes)
    steps, lr = 3, 1e-3
    tr, losses, _ = _run_trainer(wl, inp, [(0, "f32")], steps, lr)
    ref, ref_losses = O.train(inp["a"], inp["target"], inp["params"], wl.modes, [(0, "f32")],
                              steps, lr)
    np.testing.assert_allclose(losses, ref_losses, rtol=1e-4)
    assert rel_l2(_flat(tr.params()), _flat(ref)) < 1e-3


def test_trainer_precision_switch_matches_oracle():
    wl, inp = _network("bf16")
    phases, steps, lr = [(0, "bf16"), (2, "f32")], 4, 1e-3
    tr, losses, dtypes = _run_trainer(wl, inp, phases, steps, lr)
    assert dtypes == ["bf16", "bf16", "f32", "f32"]
    assert tr.dtype == "f32" and str(tr.weights.dtype) == "torch.float32"
    ref, ref_losses = O.train(inp["a"], inp["target"], inp["params"], wl.modes, phases, steps, lr)
    np.testing.assert_allclose(losses, ref_losses, rtol=2e-2)
    assert rel_l2(_flat(tr.params()), _flat(ref)) < 1e-2
