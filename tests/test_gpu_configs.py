"""Parity at the five workloads' full sizes, in the launch configuration the
benchmark uses (tensor-core kernels, library-sized workspaces).

Where the oracle cannot process the whole batch in seconds, outputs are
compared on sampled samples (every sample is independent through the whole
network) and batch-summed gradients are checked through the property that
holds at any size: the full-batch gradient equals the sum of single-sample
gradients taken with the same output cotangent.

Tolerances: relative L2 1e-5 for float32 storage, 1e-2 for 16-bit storage."""

import numpy as np
import pytest

import oracle as O
from fourier_neural_spectral_fno_b200 import capi, synth

from fno_testlib import (TOL, assert_close, dev, dev_complex, empty, host, host_complex,
                         params_to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def tensor_cores():
    capi.fno_set_tensor_cores(True)
    yield
    capi.fno_device_error(clear=True)


def _net_desc(wl, batch=None):
    return capi.net_desc(batch or wl.batch, wl.grid, wl.modes, wl.in_ch, wl.width, wl.hidden,
                         wl.out_ch, wl.n_layers, wl.dtype,
                         capi.FNO_TANH_PREACT if wl.tanh else 0)


def _run_forward(wl, a_np, params_dev, batch, saves=False):
    import torch
    d = _net_desc(wl, batch)
    u = empty((batch, wl.out_ch) + wl.grid, wl.dtype)
    sv = torch.empty(capi.fno_net_saves_size(d), dtype=torch.uint8, device="cuda") if saves else None
    capi.fno_forward(d, dev(a_np, wl.dtype), capi.make_params(params_dev), u, sv)
    return u, sv


# --------------------------------------------------------------------------
# single 2D block, float32, B4 C20 64^2 modes 12^2 (whole batch vs oracle)
# --------------------------------------------------------------------------

def test_block2d_f32_b4_w20_64sq_m12_forward_and_backward():
    wl = synth.WORKLOADS["block2d_f32_b4_w20_64sq_m12"]
    inp = synth.make_block_inputs(wl)
    x, r, w, b = inp["x"], inp["R"], inp["W"], inp["b"]
    d = capi.block_desc(wl.batch, wl.width, wl.width, wl.grid, wl.modes, wl.dtype)
    k = capi.num_modes(wl.grid, wl.modes)
    y = empty(x.shape)
    pre = empty(x.shape)
    xh = empty((wl.batch, wl.width, k, 2))
    capi.fno_block_fwd(d, dev(x), dev_complex(r), dev(w), dev(b), y, pre, xh)
    y_ref, pre_ref, xh_ref = O.block_fwd(x, r, w, b, wl.modes)
    assert_close(host(y), y_ref, TOL["f32"], "y")
    # backward with a seeded cotangent
    dy = synth.quantize(np.random.default_rng(synth.SEED_COTANGENT).standard_normal(x.shape), "f32")
    dx, dr, dw, db = empty(x.shape), empty((wl.width, wl.width, k, 2)), empty((wl.width, wl.width)), \
        empty((wl.width,))
    capi.fno_block_bwd(d, dev(x), dev_complex(r), dev(w), pre, xh, dev(dy), dx, dr, dw, db)
    # the oracle's backward takes its own forward's pre-activation, rounded to float32
    dx_ref, dr_ref, dw_ref, db_ref = O.block_bwd(x, r, w, synth.quantize(pre_ref, "f32"), xh_ref,
                                                 dy, wl.modes)
    assert_close(host(dx), dx_ref, TOL["f32"], "dx")
    assert_close(host_complex(dr), dr_ref, TOL["f32"], "dR")
    assert_close(host(dw), dw_ref, TOL["f32"], "dW")
    assert_close(host(db), db_ref, TOL["f32"], "db")


# --------------------------------------------------------------------------
# 2D FNO forward, float32, B16 width 32, 256^2, modes 16^2 (the benchmark)
# --------------------------------------------------------------------------

def test_fno2d_f32_b16_w32_256sq_m16_forward_sampled():
    wl = synth.WORKLOADS["fno2d_f32_b16_w32_256sq_m16"]
    inp = synth.make_network_inputs(wl)
    pd = params_to_device(inp["params"], wl.dtype)
    u, _ = _run_forward(wl, inp["a"], pd, wl.batch)
    got = host(u)
    for s in (0, wl.batch - 1):
        ref = O.forward(inp["a"][s:s + 1], inp["params"], wl.modes)
        assert_close(got[s:s + 1], ref, TOL["f32"], f"u[{s}]")
    assert np.all(np.isfinite(got))


def test_fno2d_forward_is_batch_independent():
    """A sample's output does not depend on the rest of the batch (any size)."""
    wl = synth.WORKLOADS["fno2d_f32_b16_w32_256sq_m16"]
    inp = synth.make_network_inputs(wl)
    pd = params_to_device(inp["params"], wl.dtype)
    u_full, _ = _run_forward(wl, inp["a"], pd, wl.batch)
    u_one, _ = _run_forward(wl, inp["a"][5:6], pd, 1)
    assert_close(host(u_one), host(u_full)[5:6], 1e-6, "u[5] alone vs in batch")


# --------------------------------------------------------------------------
# 2D block, float16 storage + tanh pre-activation, B8 C64 512^2 modes 32^2
# --------------------------------------------------------------------------

def test_block2d_f16tanh_b8_w64_512sq_m32_forward_backward():
    """Whole batch against the oracle: y and dx of every sample, and the
    batch-summed dR, dW and db against the oracle's (its per-sample backward
    passes summed).  Both backward passes take the same saved pre-activation,
    the oracle's, rounded to float16."""
    wl = synth.WORKLOADS["block2d_f16tanh_b8_w64_512sq_m32"]
    inp = synth.make_block_inputs(wl)
    x, r, w, b, dy = inp["x"], inp["R"], inp["W"], inp["b"], inp["dy"]
    fl = capi.FNO_TANH_PREACT
    C, k, B = wl.width, capi.num_modes(wl.grid, wl.modes), wl.batch
    d = capi.block_desc(B, C, C, wl.grid, wl.modes, "f16", fl)
    xd, rd, wd, bd = dev(x, "f16"), dev_complex(r, "f16"), dev(w, "f16"), dev(b, "f16")
    y, pre = empty((B, C) + wl.grid, "f16"), empty((B, C) + wl.grid, "f16")
    capi.fno_block_fwd(d, xd, rd, wd, bd, y, pre)
    yh = host(y)
    pre_q = np.empty(x.shape)
    dx_ref = np.empty(x.shape)
    dr_ref, dw_ref, db_ref = 0, 0, 0
    for s in range(B):
        y_ref, pre_ref, xh_ref = O.block_fwd(x[s:s + 1], r, w, b, wl.modes, O.TANH_PREACT)
        assert_close(yh[s:s + 1], y_ref, TOL["f16"], f"y[{s}]")
        pre_q[s:s + 1] = synth.quantize(pre_ref, "f16")
        dxs, drs, dws, dbs = O.block_bwd(x[s:s + 1], r, w, pre_q[s:s + 1], xh_ref, dy[s:s + 1],
                                         wl.modes, O.TANH_PREACT)
        dx_ref[s:s + 1] = dxs
        dr_ref, dw_ref, db_ref = dr_ref + drs, dw_ref + dws, db_ref + dbs
    dx = empty((B, C) + wl.grid, "f16")
    dr, dw, db = empty((C, C, k, 2)), empty((C, C)), empty((C,))
    capi.fno_block_bwd(d, xd, rd, wd, dev(pre_q, "f16"), None, dev(dy, "f16"), dx, dr, dw, db)
    dxh = host(dx)
    for s in range(B):
        assert_close(dxh[s:s + 1], dx_ref[s:s + 1], TOL["f16"], f"dx[{s}]")
    assert_close(host_complex(dr), dr_ref, TOL["f16"], "dR (batch of 8)")
    assert_close(host(dw), dw_ref, TOL["f16"], "dW (batch of 8)")
    assert_close(host(db), db_ref, TOL["f16"], "db (batch of 8)")


# --------------------------------------------------------------------------
# 3D FNO forward, float32, B2 width 20, 128^3, modes 8^3
# --------------------------------------------------------------------------

def test_fno3d_f32_b2_w20_128cube_m8_forward_sampled():
    wl = synth.WORKLOADS["fno3d_f32_b2_w20_128cube_m8"]
    inp = synth.make_network_inputs(wl)
    a, p = inp["a"], inp["params"]
    pd = params_to_device(p, wl.dtype)
    d = _net_desc(wl)
    u, sv = _run_forward(wl, a, pd, wl.batch, saves=True)
    # oracle for sample 0: lift and the four blocks on the whole grid, the
    # (pointwise) projection on sampled points
    v = O.lift(a[0:1], p["P"], p["p"])
    for l in range(wl.n_layers):
        v, _, _ = O.block_fwd(v, p["R"][l], p["W"][l], p["b"][l], wl.modes)
    idx = np.random.default_rng(11).choice(wl.points, 4096, replace=False)
    v_pts = v.reshape(1, wl.width, -1)[:, :, idx]
    u_ref = O.projection(v_pts, p["Q1"], p["q1"], p["Q2"], p["q2"])
    got = host(u)[0:1].reshape(1, 1, -1)[:, :, idx]
    assert_close(got, u_ref, TOL["f32"], "u[0] sampled points")
    # the last block's output (kept in the saves) on the whole grid
    import ctypes
    saves = sv.cpu().numpy()
    act = wl.batch * wl.width * wl.points * 4
    act_al = (act + 255) // 256 * 256
    xh_al = (wl.batch * wl.width * capi.num_modes(wl.grid, wl.modes) * 8 + 255) // 256 * 256
    off = wl.n_layers * (2 * act_al + xh_al)
    v_gpu = saves[off:off + act].view(np.float32).reshape((wl.batch, wl.width) + wl.grid)
    assert_close(v_gpu[0:1].astype(np.float64), v, TOL["f32"], "v_L[0]")
    del ctypes, d


# --------------------------------------------------------------------------
# 2D FNO training step, bfloat16 storage, B32 width 64, 256^2, modes 24^2
# --------------------------------------------------------------------------

def test_fno2d_bf16_train_b32_w64_256sq_m24_step():
    import torch
    wl = synth.WORKLOADS["fno2d_bf16_train_b32_w64_256sq_m24"]
    inp = synth.make_network_inputs(wl)
    a, p, tgt = inp["a"], inp["params"], inp["target"]
    pd = params_to_device(p, "bf16")
    cp = capi.make_params(pd)

    def step(lo, hi, du_in=None):
        n = hi - lo
        d = _net_desc(wl, n)
        u = empty((n, 1) + wl.grid, "bf16")
        sv = torch.empty(capi.fno_net_saves_size(d), dtype=torch.uint8, device="cuda")
        ad = dev(a[lo:hi], "bf16")
        capi.fno_forward(d, ad, cp, u, sv)
        loss = torch.empty(1, dtype=torch.float32, device="cuda")
        du = empty(u.shape, "bf16")
        capi.fno_mse(u, dev(tgt[lo:hi], "bf16"), loss, du, "bf16")
        if du_in is not None:
            du = du_in
        g = {k: ([torch.empty(v.shape + ((2,) if np.iscomplexobj(v) else ()), device="cuda")
                  for v in vals] if isinstance(vals, list)
                 else torch.empty(np.shape(vals), device="cuda")) for k, vals in p.items()}
        capi.fno_backward(d, ad, cp, sv, du, capi.make_grads(g))
        return u, loss, du, g

    u, loss, du, g = step(0, wl.batch)
    uh = host(u)
    # loss against the MSE of the stored output
    ref_loss = float(np.mean((uh - tgt) ** 2))
    assert abs(loss.item() - ref_loss) <= 1e-3 * ref_loss
    # per-sample outputs against the oracle
    for s in (0, wl.batch - 1):
        u_ref = O.forward(a[s:s + 1], p, wl.modes)
        assert_close(uh[s:s + 1], u_ref, TOL["bf16"], f"u[{s}]")
    # gradients of sample 0 against the oracle, both sides fed the oracle's
    # cotangent: dL/du of the full-batch MSE restricted to sample 0, in bfloat16
    u_ref, sv_ref = O.forward(a[0:1], p, wl.modes, save=True)
    du0_ref = synth.quantize(2.0 * (u_ref - tgt[0:1]) / tgt.size, "bf16")
    _, _, _, g0 = step(0, 1, dev(du0_ref, "bf16"))
    g_ref = O.backward(a[0:1], p, sv_ref, du0_ref, wl.modes)
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        assert_close(host(g0[key]), g_ref[key], TOL["bf16"], f"d{key} (sample 0)")
    for l in range(wl.n_layers):
        assert_close(host_complex(g0["R"][l]), g_ref["R"][l], TOL["bf16"], f"dR[{l}] (sample 0)")
        assert_close(host(g0["W"][l]), g_ref["W"][l], TOL["bf16"], f"dW[{l}] (sample 0)")
        assert_close(host(g0["b"][l]), g_ref["b"][l], TOL["bf16"], f"db[{l}] (sample 0)")

    # every full-batch gradient equals the sum of the single-sample gradients
    # taken with the same cotangent (each sample is independent)
    def flat(g):
        out = [(k, host(g[k])) for k in ("P", "p", "Q1", "q1", "Q2", "q2")]
        for l in range(wl.n_layers):
            out += [(f"R[{l}]", host_complex(g["R"][l])), (f"W[{l}]", host(g["W"][l])),
                    (f"b[{l}]", host(g["b"][l]))]
        return out

    acc = None
    for s in range(wl.batch):
        _, _, _, gs = step(s, s + 1, du[s:s + 1].clone())
        fs = flat(gs)
        acc = fs if acc is None else [(k, x + y) for (k, x), (_, y) in zip(acc, fs)]
    for (k, x), (_, y) in zip(flat(g), acc):
        assert_close(x, y, 1e-4, f"d{k}: full batch = sum of samples")
