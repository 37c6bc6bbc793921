"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by
element, on seeded inputs at sizes that span several tiles and ragged tails.

Tolerances: relative L2 error 1e-5 for float32 storage, 1e-2 for float16 /
bfloat16 storage with float32 accumulation."""

import numpy as np
import pytest

import oracle as O
from fourier_neural_spectral_fno_b200 import capi, synth

from fno_testlib import (TOL, assert_close, dev, dev_complex, empty, flags_of, grads_like, host,
                         host_complex, oracle_flags, params_to_device)

pytestmark = pytest.mark.gpu

# (grid, modes): 1D, 2D with ragged row tiles / column chunks, odd lengths, all
# modes kept, 3D with ragged slabs
SHAPES = [
    ((100,), (20,)),
    ((16, 12), (4, 5)),
    ((15, 9), (5, 5)),
    ((8, 8), (4, 5)),
    ((70, 130), (6, 9)),
    ((6, 10, 12), (2, 3, 4)),
    ((20, 9, 70), (5, 4, 11)),
    # shapes the tensor-core kernels take (128-byte rows, 128-row / 128-point tiles)
    ((64, 64), (10, 12)),
    ((256, 128), (16, 20)),
    ((32, 96), (8, 16)),
    ((8, 16, 64), (2, 4, 8)),
    ((128,), (30,)),
    ((384, 64), (40, 33)),
    # shapes the pipelined forward transform takes (128-row bands, 128-byte
    # column chunks, <= 16 last-axis and <= 32 slab-axis modes); 96-wide rows
    # are whole chunks in float32 only
    ((128, 64), (8, 8)),
    ((256, 96), (16, 12)),
    ((384, 128), (10, 16)),
    ((4, 128, 64), (2, 8, 8)),
    # shapes the pruned-FFT transform takes (last axis 64, 128, 256 or 512 with
    # at most 32 modes): ragged slab bands, several-CTA clusters, the fused
    # spectral middle (slab axis a multiple of 16) and its fallback
    ((40, 256), (7, 16)),
    ((48, 512), (9, 32)),
    ((272, 64), (30, 5)),
    ((1100, 64), (3, 8)),
    ((96, 128), (20, 24)),
    ((6, 32, 128), (3, 4, 9)),
]


@pytest.fixture(autouse=True, params=[1, 4, 3, 2, 0],
                ids=["default", "fft_cluster", "tc_dft", "tc_nopipe", "cudacore"])
def kernel_path(request):
    """Every parity test runs on the default kernels (streaming pruned-FFT
    transform, mixing and pruned slab-axis inverse, tcgen05 epilogue
    pipeline), on the default with the clustered FFT transform, on the tcgen05
    TMA pipelines with the dense DFT-matrix transform, on the tcgen05 kernels
    without pipelines (where the shape allows each) and on the CUDA-core
    kernels; no bounded device wait may expire."""
    capi.fno_set_tensor_cores(request.param)
    yield request.param
    capi.fno_device_error(clear=True)
    capi.fno_set_tensor_cores(True)


def _block_inputs(grid, modes, batch, ci, co, dtype, seed=0, bias=True):
    rng = np.random.default_rng(seed)
    x = synth.quantize(rng.standard_normal((batch, ci) + tuple(grid)), dtype)
    k = capi.num_modes(grid, modes)
    r = synth.quantize_complex(synth.spectral_weights(rng, ci, co, k) * (ci * co) / np.sqrt(ci), dtype)
    w = synth.quantize(rng.uniform(-1, 1, (co, ci)) / np.sqrt(ci), dtype)
    b = synth.quantize(rng.uniform(-0.5, 0.5, co) if bias else np.zeros(co), dtype)
    dy = synth.quantize(rng.standard_normal((batch, co) + tuple(grid)), dtype)
    return x, r, w, b, dy


@pytest.mark.parametrize("grid,modes", SHAPES)
@pytest.mark.parametrize("dtype,tanh", [("f32", False), ("f32", True), ("f16", True),
                                        ("bf16", False)])
def test_spectral_conv_fwd(grid, modes, dtype, tanh):
    b_, ci, co = 3, 5, 4
    x, r, _, _, _ = _block_inputs(grid, modes, b_, ci, co, dtype)
    flags = flags_of(tanh=tanh)
    d = capi.block_desc(b_, ci, co, grid, modes, dtype, flags)
    k = capi.num_modes(grid, modes)
    y = empty((b_, co) + grid, dtype)
    xh = empty((b_, ci, k, 2))
    capi.fno_spectral_conv_fwd(d, dev(x, dtype), dev_complex(r, dtype), y, xh)
    y_ref, xh_ref = O.spectral_conv_fwd(x, r, modes, oracle_flags(flags))
    # 16-bit storage: the transform runs with 16-bit operands (float32 accumulation)
    assert_close(host_complex(xh), xh_ref, TOL[dtype], "xhat")
    assert_close(host(y), y_ref, TOL[dtype], "y")


@pytest.mark.parametrize("grid,modes", SHAPES)
@pytest.mark.parametrize("dtype,flags", [("f32", 0), ("f32", 2), ("f16", 1), ("bf16", 0)])
def test_block_fwd(grid, modes, dtype, flags):
    b_, ci, co = 2, 6, 7
    x, r, w, b, _ = _block_inputs(grid, modes, b_, ci, co, dtype, seed=1)
    d = capi.block_desc(b_, ci, co, grid, modes, dtype, flags)
    k = capi.num_modes(grid, modes)
    y = empty((b_, co) + grid, dtype)
    pre = empty((b_, co) + grid, dtype)
    xh = empty((b_, ci, k, 2))
    capi.fno_block_fwd(d, dev(x, dtype), dev_complex(r, dtype), dev(w, dtype), dev(b, dtype), y,
                       pre, xh)
    y_ref, pre_ref, xh_ref = O.block_fwd(x, r, w, b, modes, oracle_flags(flags))
    assert_close(host(pre), pre_ref, TOL[dtype], "pre")
    assert_close(host(y), y_ref, TOL[dtype], "y")
    assert_close(host_complex(xh), xh_ref, TOL[dtype], "xhat")


@pytest.mark.parametrize("grid,modes", SHAPES)
@pytest.mark.parametrize("dtype,tanh,give_xhat", [("f32", False, True), ("f32", True, False),
                                                  ("f16", True, True), ("bf16", False, False)])
def test_spectral_conv_bwd(grid, modes, dtype, tanh, give_xhat):
    b_, ci, co = 3, 4, 5
    x, r, _, _, dy = _block_inputs(grid, modes, b_, ci, co, dtype, seed=2)
    flags = flags_of(tanh=tanh)
    d = capi.block_desc(b_, ci, co, grid, modes, dtype, flags)
    k = capi.num_modes(grid, modes)
    _, xh_ref = O.spectral_conv_fwd(x, r, modes, oracle_flags(flags))
    xh = dev_complex(xh_ref) if give_xhat else None
    dx = empty((b_, ci) + grid, dtype)
    dr = empty((ci, co, k, 2))
    capi.fno_spectral_conv_bwd(d, dev(x, dtype), xh, dev_complex(r, dtype), dev(dy, dtype), dx, dr)
    dx_ref, dr_ref = O.spectral_conv_bwd(x, r, xh_ref, dy, modes, oracle_flags(flags))
    assert_close(host(dx), dx_ref, TOL[dtype], "dx")
    assert_close(host_complex(dr), dr_ref, TOL[dtype] if dtype != "f32" else 1e-5, "dR")


@pytest.mark.parametrize("grid,modes", SHAPES)
@pytest.mark.parametrize("dtype,flags,give_xhat", [("f32", 0, True), ("f32", 1, False),
                                                   ("f32", 2, True), ("f16", 1, True),
                                                   ("bf16", 0, False)])
def test_block_bwd(grid, modes, dtype, flags, give_xhat):
    b_, ci, co = 2, 5, 6
    x, r, w, b, dy = _block_inputs(grid, modes, b_, ci, co, dtype, seed=3)
    d = capi.block_desc(b_, ci, co, grid, modes, dtype, flags)
    k = capi.num_modes(grid, modes)
    y_ref, pre_ref, xh_ref = O.block_fwd(x, r, w, b, modes, oracle_flags(flags))
    pre_q = synth.quantize(pre_ref, dtype)          # what the forward saved
    dx = empty((b_, ci) + grid, dtype)
    dr = empty((ci, co, k, 2))
    dw = empty((co, ci))
    db = empty((co,))
    capi.fno_block_bwd(d, dev(x, dtype), dev_complex(r, dtype), dev(w, dtype), dev(pre_q, dtype),
                       dev_complex(xh_ref) if give_xhat else None, dev(dy, dtype), dx, dr, dw, db)
    dx_ref, dr_ref, dw_ref, db_ref = O.block_bwd(x, r, w, pre_q, xh_ref, dy, modes,
                                                 oracle_flags(flags))
    tol = TOL[dtype]
    assert_close(host(dx), dx_ref, tol, "dx")
    assert_close(host_complex(dr), dr_ref, tol, "dR")
    assert_close(host(dw), dw_ref, tol, "dW")
    assert_close(host(db), db_ref, tol, "db")


@pytest.mark.parametrize("grid,modes,batch", [((32, 32), (8, 8), 3), ((64, 48), (10, 12), 33),
                                              ((32, 32), (8, 8), 64), ((15, 9), (5, 5), 20)])
@pytest.mark.parametrize("ci,co", [(64, 64), (16, 64), (64, 40)])
def test_mixing_64_channels_bf16(grid, modes, batch, ci, co):
    """The tensor-core mixing (bfloat16 weights, 64 output channels of the
    forward or of the adjoint dxhat; batch padded to the MMA's N) against the
    oracle, through the spectral forward and backward; the last shape (K not a
    multiple of four) and the channel pairs without 64 outputs take the CUDA
    cores."""
    x, r, _, _, dy = _block_inputs(grid, modes, batch, ci, co, "bf16", seed=5)
    d = capi.block_desc(batch, ci, co, grid, modes, "bf16")
    k = capi.num_modes(grid, modes)
    y = empty((batch, co) + grid, "bf16")
    xh = empty((batch, ci, k, 2))
    capi.fno_spectral_conv_fwd(d, dev(x, "bf16"), dev_complex(r, "bf16"), y, xh)
    y_ref, xh_ref = O.spectral_conv_fwd(x, r, modes)
    assert_close(host(y), y_ref, TOL["bf16"], "y")
    dx = empty((batch, ci) + grid, "bf16")
    dr = empty((ci, co, k, 2))
    capi.fno_spectral_conv_bwd(d, dev(x, "bf16"), dev_complex(xh_ref), dev_complex(r, "bf16"),
                               dev(dy, "bf16"), dx, dr)
    dx_ref, dr_ref = O.spectral_conv_bwd(x, r, xh_ref, dy, modes)
    assert_close(host(dx), dx_ref, TOL["bf16"], "dx")
    assert_close(host_complex(dr), dr_ref, TOL["bf16"], "dR")


def test_block_bwd_wide_channels_f32():
    grid, modes = (32, 40), (5, 7)
    x, r, w, b, dy = _block_inputs(grid, modes, 3, 64, 48, "f32", seed=4)
    d = capi.block_desc(3, 64, 48, grid, modes)
    y_ref, pre_ref, xh_ref = O.block_fwd(x, r, w, b, modes)
    y = empty((3, 48) + grid)
    pre = empty((3, 48) + grid)
    capi.fno_block_fwd(d, dev(x), dev_complex(r), dev(w), dev(b), y, pre)
    assert_close(host(y), y_ref, 1e-5, "y")
    k = capi.num_modes(grid, modes)
    dx, dr, dw, db = empty((3, 64) + grid), empty((64, 48, k, 2)), empty((48, 64)), empty((48,))
    # both sides take the same saved pre-activation: the oracle's, rounded to float32
    pre_q = synth.quantize(pre_ref, "f32")
    capi.fno_block_bwd(d, dev(x), dev_complex(r), dev(w), dev(pre_q), None, dev(dy), dx, dr, dw, db)
    dx_ref, dr_ref, dw_ref, db_ref = O.block_bwd(x, r, w, pre_q, xh_ref, dy, modes)
    assert_close(host(dx), dx_ref, 1e-5, "dx")
    assert_close(host_complex(dr), dr_ref, 1e-5, "dR")
    assert_close(host(dw), dw_ref, 1e-5, "dW")
    assert_close(host(db), db_ref, 1e-5, "db")


def _tiny_network(grid, modes, dtype, batch=2, width=6, hidden=9, layers=2, in_ch=None):
    in_ch = in_ch or 1 + len(grid)
    wl = synth.Workload("tiny", "network", dtype, batch, tuple(grid), tuple(modes), width,
                        in_ch=in_ch, hidden=hidden, n_layers=layers, backward=True)
    inp = synth.make_network_inputs(wl)
    p = inp["params"]
    p["R"] = [synth.quantize_complex(r * width * width / np.sqrt(width), dtype) for r in p["R"]]
    p["b"] = [synth.quantize(np.linspace(-0.3, 0.3, width), dtype) for _ in p["b"]]
    return wl, inp


@pytest.mark.parametrize("grid,modes", [((16, 12), (4, 5)), ((40, 70), (6, 9)),
                                        ((6, 10, 12), (2, 3, 4)), ((100,), (20,)),
                                        ((64, 64), (10, 12)), ((8, 16, 64), (2, 4, 8)),
                                        ((256,), (40,))])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_network_forward_backward_mse(grid, modes, dtype):
    import torch
    wl, inp = _tiny_network(grid, modes, dtype)
    a, params, tgt = inp["a"], inp["params"], inp["target"]
    d = capi.net_desc(wl.batch, grid, modes, wl.in_ch, wl.width, wl.hidden, 1, wl.n_layers, dtype)
    pd = params_to_device(params, dtype)
    cp = capi.make_params(pd)
    saves = torch.empty(capi.fno_net_saves_size(d), dtype=torch.uint8, device="cuda")
    u = empty((wl.batch, 1) + grid, dtype)
    a_d = dev(a, dtype)
    capi.fno_forward(d, a_d, cp, u, saves)
    u_ref, sv = O.forward(a, params, modes, save=True)
    assert_close(host(u), u_ref, TOL[dtype], "u")
    # forward without saves gives the same result
    u2 = empty((wl.batch, 1) + grid, dtype)
    capi.fno_forward(d, a_d, cp, u2)
    assert torch.equal(u, u2)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    du = empty(u.shape, dtype)
    capi.fno_mse(u, dev(tgt, dtype), loss, du, dtype)
    loss_ref, du_ref = O.mse(host(u), tgt)
    assert abs(float(loss.item()) - loss_ref) <= 1e-5 * abs(loss_ref) + 1e-7
    assert_close(host(du), du_ref, TOL[dtype], "du")
    gd = grads_like(params)
    capi.fno_backward(d, a_d, cp, saves, du, capi.make_grads(gd))
    g_ref = O.backward(a, params, sv, host(du), modes)
    tol = TOL[dtype]
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        assert_close(host(gd[key]), g_ref[key], tol, key)
    for key in ("R", "W", "b"):
        for l in range(wl.n_layers):
            got = host_complex(gd[key][l]) if key == "R" else host(gd[key][l])
            assert_close(got, g_ref[key][l], tol, f"{key}[{l}]")


def test_default_path_launches_four_kernels_per_block():
    """On a 2D grid the default path runs a block forward as the pruned-FFT
    transform, the mixing, the pruned slab-axis inverse and the epilogue."""
    grid, modes = (256, 256), (16, 16)
    x, r, w, b, _ = _block_inputs(grid, modes, 2, 8, 8, "f32")
    d = capi.block_desc(2, 8, 8, grid, modes)
    y = empty((2, 8) + grid)
    prev = capi.fno_set_tensor_cores(1)
    try:
        capi.fno_block_fwd(d, dev(x), dev_complex(r), dev(w), dev(b), y)
        assert capi.last_launch_count() == 4
    finally:
        capi.fno_set_tensor_cores(prev)


def test_launch_count_is_reported(kernel_path):
    grid, modes = (16, 12), (4, 5)
    x, r, w, b, _ = _block_inputs(grid, modes, 2, 3, 3, "f32")
    d = capi.block_desc(2, 3, 3, grid, modes)
    y = empty((2, 3) + grid)
    capi.fno_block_fwd(d, dev(x), dev_complex(r), dev(w), dev(b), y)
    # transform, finish, mix, epilogue; the default path inverts the slab axis
    # in a launch of its own
    assert capi.last_launch_count() == (5 if kernel_path in (1, 4) else 4)


@pytest.mark.parametrize("grid,modes", [((64, 64), (10, 12)), ((256, 128), (16, 20)), ((15, 9), (5, 5))])
def test_block_gelu_elementwise(grid, modes):
    """With R = 0, W = I and b = 0 the block output is GELU(x) point by point,
    which pins the kernels' GELU elementwise (not only in the L2 norm).  Their
    erf is formula 7.1.28 of Abramowitz and Stegun (|error| <= 3e-7), so the
    GELU adds at most |x| 1.5e-7; the pre-activation W x through the three tf32
    passes is within 2^-23 |x| (the rounded remainder), and the float32
    roundings add about 1.5e-7 |x|: within 5e-7 max(1, |x|) of the exact erf
    form at every point."""
    b_, c = 2, 16
    n = int(np.prod(grid))
    x = np.linspace(-9.0, 9.0, b_ * c * n).reshape((b_, c) + tuple(grid))
    x = synth.quantize(np.random.default_rng(5).permutation(x.ravel()).reshape(x.shape), "f32")
    k = capi.num_modes(grid, modes)
    r = np.zeros((c, c, k), np.complex128)
    w = np.eye(c)
    d = capi.block_desc(b_, c, c, grid, modes)
    y = empty((b_, c) + grid)
    capi.fno_block_fwd(d, dev(x), dev_complex(r), dev(w), dev(np.zeros(c)), y)
    got = host(y).astype(np.float64)
    ref = O.gelu(x.astype(np.float64))
    err = np.abs(got - ref)
    assert np.max(err / np.maximum(np.abs(x), 1.0)) < 5e-7


def _cp_inputs(grid, modes, rank, ci, co, dtype, seed):
    rng = np.random.default_rng(seed)
    k = capi.num_modes(grid, modes)

    def cplx(*shape):
        return synth.quantize_complex(rng.uniform(-1, 1, shape) + 1j * rng.uniform(-1, 1, shape),
                                      dtype)
    lam = cplx(rank)
    a, b, c = cplx(ci, rank), cplx(co, rank), cplx(k, rank)
    return lam, a, b, c


@pytest.mark.parametrize("grid,modes", [((64, 64), (10, 12)), ((15, 9), (5, 5)),
                                        ((256, 256), (16, 16)), ((6, 10, 12), (2, 3, 4))])
@pytest.mark.parametrize("rank", [1, 5, 16, 32])
@pytest.mark.parametrize("dtype,flags", [("f32", 0), ("f16", 1), ("bf16", 0)])
def test_factorised_weights_forward(grid, modes, rank, dtype, flags):
    """CP-factorised weights against the oracle's dense reconstruction: the
    spectral forward (spectral_conv_fwd_cp) and the block forward (block_fwd
    with R = cp_weights)."""
    b_, ci, co = 2, 6, 5
    x, _, w, b, _ = _block_inputs(grid, modes, b_, ci, co, dtype, seed=7)
    lam, a, bf, c = _cp_inputs(grid, modes, rank, ci, co, dtype, seed=8)
    d = capi.block_desc(b_, ci, co, grid, modes, dtype, flags)
    k = capi.num_modes(grid, modes)
    dv = [dev_complex(v, dtype) for v in (lam, a, bf, c)]
    y = empty((b_, co) + grid, dtype)
    xh = empty((b_, ci, k, 2))
    capi.fno_spectral_conv_fwd_cp(d, rank, dev(x, dtype), *dv, y, xh)
    y_ref, xh_ref = O.spectral_conv_fwd_cp(x, lam, a, bf, c, modes, oracle_flags(flags))
    assert_close(host_complex(xh), xh_ref, TOL[dtype], "xhat")
    assert_close(host(y), y_ref, TOL[dtype], "y (spectral)")
    yb, pre = empty((b_, co) + grid, dtype), empty((b_, co) + grid, dtype)
    capi.fno_block_fwd_cp(d, rank, dev(x, dtype), *dv, dev(w, dtype), dev(b, dtype), yb, pre)
    yb_ref, pre_ref, _ = O.block_fwd(x, O.cp_weights(lam, a, bf, c), w, b, modes,
                                     oracle_flags(flags))
    assert_close(host(pre), pre_ref, TOL[dtype], "pre (block)")
    assert_close(host(yb), yb_ref, TOL[dtype], "y (block)")


@pytest.mark.parametrize("grid,modes", [((64, 64), (10, 12)), ((15, 9), (5, 5)),
                                        ((256, 256), (16, 16)), ((6, 10, 12), (2, 3, 4))])
@pytest.mark.parametrize("rank", [1, 7, 32])
@pytest.mark.parametrize("dtype,flags", [("f32", 0), ("f32", 1), ("bf16", 0)])
def test_factorised_weights_backward(grid, modes, rank, dtype, flags):
    """Adjoints through the CP factors against the oracle: dx and the factor
    gradients of the spectral convolution (spectral_conv_bwd_cp), and of the
    block (block_bwd on cp_weights, then cp_factor_grads)."""
    import torch
    b_, ci, co = 2, 5, 6
    x, _, w, b, dy = _block_inputs(grid, modes, b_, ci, co, dtype, seed=9)
    fac = _cp_inputs(grid, modes, rank, ci, co, dtype, seed=10)
    d = capi.block_desc(b_, ci, co, grid, modes, dtype, flags)
    k = capi.num_modes(grid, modes)
    dv = [dev_complex(v, dtype) for v in fac]
    of = oracle_flags(flags)
    _, xh_ref = O.spectral_conv_fwd_cp(x, *fac, modes, of)
    outs = [empty((b_, ci) + grid, dtype), empty((rank, 2)), empty((ci, rank, 2)),
            empty((co, rank, 2)), empty((k, rank, 2))]
    capi.fno_spectral_conv_bwd_cp(d, rank, dev(x, dtype), *dv, dev_complex(xh_ref), dev(dy, dtype),
                                  *outs)
    ref = O.spectral_conv_bwd_cp(x, *fac, xh_ref, dy, modes, of)
    assert_close(host(outs[0]), ref[0], TOL[dtype], "dx (spectral)")
    for name, got, want in zip(("dlam", "dA", "dB", "dC"), outs[1:], ref[1:]):
        assert_close(host_complex(got), want, TOL[dtype], name + " (spectral)")
    # the block: the oracle forward's pre-activation, rounded to the storage dtype, on both sides
    r_dense = O.cp_weights(*fac)
    _, pre_ref, _ = O.block_fwd(x, r_dense, w, b, modes, of)
    pre_q = synth.quantize(pre_ref, dtype)
    outs = [empty((b_, ci) + grid, dtype), empty((rank, 2)), empty((ci, rank, 2)),
            empty((co, rank, 2)), empty((k, rank, 2)), empty((co, ci)), empty((co,))]
    capi.fno_block_bwd_cp(d, rank, dev(x, dtype), *dv, dev(w, dtype), dev(pre_q, dtype), None,
                          dev(dy, dtype), *outs)
    dx_ref, dr_ref, dw_ref, db_ref = O.block_bwd(x, r_dense, w, pre_q, xh_ref, dy, modes, of)
    dfac = O.cp_factor_grads(dr_ref, *fac)
    assert_close(host(outs[0]), dx_ref, TOL[dtype], "dx (block)")
    for name, got, want in zip(("dlam", "dA", "dB", "dC"), outs[1:5], dfac):
        assert_close(host_complex(got), want, TOL[dtype], name + " (block)")
    assert_close(host(outs[5]), dw_ref, TOL[dtype], "dW (block)")
    assert_close(host(outs[6]), db_ref, TOL[dtype], "db (block)")
    del torch


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_replays_as_cuda_graph(dtype):
    """The network forward allocates nothing and never synchronises, so it can be
    captured into a CUDA graph: every replay equals the eager call bit for bit,
    including after the input is rewritten in place (the graph reads the buffers,
    not copies of them), and the replay matches the oracle."""
    import torch
    grid, modes = (256, 256), (16, 16)
    wl, inp = _tiny_network(grid, modes, dtype, batch=2, width=32, hidden=128, layers=4, in_ch=3)
    d = capi.net_desc(wl.batch, grid, modes, wl.in_ch, wl.width, wl.hidden, 1, wl.n_layers, dtype)
    pd = params_to_device(inp["params"], dtype)    # kept alive: cp holds raw pointers
    cp = capi.make_params(pd)
    ws = torch.empty(capi.fno_net_workspace_size(d, capi.FNO_OP_NET_FWD), dtype=torch.uint8,
                     device="cuda")
    a_d = dev(inp["a"], dtype)
    u_eager = empty((wl.batch, 1) + grid, dtype)
    u_graph = empty((wl.batch, 1) + grid, dtype)
    capi.fno_forward(d, a_d, cp, u_eager, None, ws, torch.cuda.current_stream())
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        capi.fno_forward(d, a_d, cp, u_graph, None, ws, torch.cuda.current_stream())
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(u_graph, u_eager)
    a2 = np.random.default_rng(7).standard_normal(inp["a"].shape)
    a2 = synth.quantize(a2, dtype)
    a_d.copy_(dev(a2, dtype))
    g.replay()
    capi.fno_forward(d, a_d, cp, u_eager, None, ws, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert torch.equal(u_graph, u_eager)
    assert_close(host(u_graph), O.forward(a2, inp["params"], modes), TOL[dtype], "u")
