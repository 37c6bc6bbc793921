"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
function include/fno.h declares, its structs have the C layout, and argument
validation rejects bad calls before anything is enqueued."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from fourier_neural_spectral_fno_b200 import build, capi, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fno.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fno_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(capi.EXPORTED) == names


def test_version_string(lib):
    assert b"sm_100a" in lib.fno_version()


LAYOUT_PROG = r"""
#include <stdio.h>
#include <stddef.h>
#include "fno.h"
#define F(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  printf("fno_block_desc %zu\n", sizeof(fno_block_desc));
  F(fno_block_desc, ndim) F(fno_block_desc, dtype) F(fno_block_desc, flags) F(fno_block_desc, cin)
  F(fno_block_desc, cout) F(fno_block_desc, batch) F(fno_block_desc, grid) F(fno_block_desc, modes)
  printf("fno_net_desc %zu\n", sizeof(fno_net_desc));
  F(fno_net_desc, in_channels) F(fno_net_desc, width) F(fno_net_desc, hidden)
  F(fno_net_desc, out_channels) F(fno_net_desc, n_layers) F(fno_net_desc, batch)
  F(fno_net_desc, grid) F(fno_net_desc, modes)
  printf("fno_params %zu\n", sizeof(fno_params));
  F(fno_params, P) F(fno_params, p) F(fno_params, R) F(fno_params, W) F(fno_params, b)
  F(fno_params, Q1) F(fno_params, q1) F(fno_params, Q2) F(fno_params, q2)
  printf("fno_grads %zu\n", sizeof(fno_grads));
  F(fno_grads, R) F(fno_grads, q2)
  return 0;
}
"""


def test_struct_layout_matches_c():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(src, "w").write(LAYOUT_PROG)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    got = dict(line.rsplit(" ", 1) for line in out.strip().splitlines())
    cls = {"fno_block_desc": capi.BlockDesc, "fno_net_desc": capi.NetDesc,
           "fno_params": capi.Params, "fno_grads": capi.Grads}
    for key, val in got.items():
        if "." in key:
            s, f = key.split(".")
            assert getattr(cls[s], f).offset == int(val), key
        else:
            assert ctypes.sizeof(cls[key]) == int(val), key


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER)
def test_workspace_sizes_for_every_workload(lib, name):
    wl = synth.WORKLOADS[name]
    flags = capi.FNO_TANH_PREACT if wl.tanh else 0
    if wl.kind == "block":
        d = capi.block_desc(wl.batch, wl.width, wl.width, wl.grid, wl.modes, wl.dtype, flags)
        for op in (0, 1, 2, 3):
            assert capi.fno_workspace_size(d, op) > 0
    else:
        d = capi.net_desc(wl.batch, wl.grid, wl.modes, wl.in_ch, wl.width, wl.hidden, wl.out_ch,
                          wl.n_layers, wl.dtype, flags)
        assert capi.fno_net_workspace_size(d, capi.FNO_OP_NET_FWD) > 0
        assert capi.fno_net_workspace_size(d, capi.FNO_OP_NET_BWD) > 0
        assert capi.fno_net_saves_size(d) > 0


@pytest.mark.parametrize("grid,modes,code", [
    ((64, 64), (33, 12), capi.FNO_ERR_INVALID_ARG),   # 2m > N on a non-last axis
    ((64, 64), (12, 34), capi.FNO_ERR_INVALID_ARG),   # m > N/2+1 on the last axis
    ((64, 64), (0, 12), capi.FNO_ERR_INVALID_ARG),
    ((8192, 64), (12, 12), capi.FNO_ERR_UNSUPPORTED),  # axis longer than the twiddle tables
    ((64, 256), (12, 100), capi.FNO_ERR_UNSUPPORTED),  # more than 64 last-axis modes
])
def test_invalid_descriptors(lib, grid, modes, code):
    d = capi.block_desc(2, 4, 4, grid, modes)
    assert lib.fno_workspace_size(ctypes.byref(d), capi.FNO_OP_BLOCK_FWD) == 0
    rc = lib.fno_block_fwd(ctypes.byref(d), 256, 256, 256, 256, 256, None, None, 256, 1 << 30, None)
    assert rc == code, capi.last_error()
    assert capi.last_error()


def test_invalid_channels_and_dtype(lib):
    d = capi.block_desc(2, 0, 4, (16, 16), (4, 4))
    assert lib.fno_block_fwd(ctypes.byref(d), 256, 256, 256, 256, 256, None, None, 256, 1 << 30,
                             None) == capi.FNO_ERR_INVALID_ARG
    d = capi.block_desc(2, 65, 4, (16, 16), (4, 4))
    assert lib.fno_block_fwd(ctypes.byref(d), 256, 256, 256, 256, 256, None, None, 256, 1 << 30,
                             None) == capi.FNO_ERR_UNSUPPORTED
    d = capi.block_desc(2, 4, 4, (16, 16), (4, 4))
    d.dtype = 7
    assert lib.fno_spectral_conv_fwd(ctypes.byref(d), 256, 256, 256, None, 256, 1 << 30,
                                     None) == capi.FNO_ERR_INVALID_ARG
    d.dtype = 0
    d.flags = 8
    assert lib.fno_spectral_conv_fwd(ctypes.byref(d), 256, 256, 256, None, 256, 1 << 30,
                                     None) == capi.FNO_ERR_INVALID_ARG
    assert lib.fno_spectral_conv_fwd(None, 256, 256, 256, None, 256, 1 << 30,
                                     None) == capi.FNO_ERR_INVALID_ARG


def test_null_misaligned_and_workspace(lib):
    d = capi.block_desc(2, 4, 4, (16, 16), (4, 4))
    need = capi.fno_workspace_size(d, capi.FNO_OP_SPECTRAL_FWD)
    f = lib.fno_spectral_conv_fwd
    assert f(ctypes.byref(d), None, 256, 256, None, 256, need, None) == capi.FNO_ERR_INVALID_ARG
    assert "x" in capi.last_error()
    assert f(ctypes.byref(d), 0x1008, 256, 256, None, 256, need, None) == capi.FNO_ERR_INVALID_ARG
    assert "aligned" in capi.last_error()
    assert f(ctypes.byref(d), 256, 256, 256, 0x104, 256, need, None) == capi.FNO_ERR_INVALID_ARG
    assert f(ctypes.byref(d), 256, 256, 256, None, 256, need - 1, None) == capi.FNO_ERR_WORKSPACE
    assert f(ctypes.byref(d), 256, 256, 256, None, None, need, None) == capi.FNO_ERR_INVALID_ARG
    bw = lib.fno_block_bwd
    assert bw(ctypes.byref(d), 256, 256, 256, None, None, 256, 256, 256, 256, 256, 256, 1 << 30,
              None) == capi.FNO_ERR_INVALID_ARG          # pre_save required with GELU
    assert "pre_save" in capi.last_error()


def test_network_validation(lib):
    d = capi.net_desc(2, (16, 16), (4, 4), 3, 8, n_layers=0)
    assert lib.fno_net_workspace_size(ctypes.byref(d), capi.FNO_OP_NET_FWD) == 0
    d = capi.net_desc(2, (16, 16), (4, 4), 3, 8, out_channels=5)
    assert lib.fno_net_saves_size(ctypes.byref(d)) == 0
    d = capi.net_desc(2, (16, 16), (4, 4), 3, 8)
    p = capi.Params()
    assert lib.fno_forward(ctypes.byref(d), 256, ctypes.byref(p), 256, None, 256, 1 << 30,
                           None) == capi.FNO_ERR_INVALID_ARG
    assert lib.fno_mse(0, 0, 256, 256, 256, None, None) == capi.FNO_ERR_INVALID_ARG


@pytest.mark.parametrize("args,word", [
    # n, theta, m, v, grad, out, out_dtype, step, lr, beta1, beta2, eps, wd, scale
    ((0, 256, 256, 256, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "n 0"),
    ((8, None, 256, 256, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "theta"),
    ((8, 0x108, 256, 256, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "aligned"),
    ((8, 256, None, 256, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "m is NULL"),
    ((8, 256, 256, None, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "v is NULL"),
    ((8, 256, 256, 256, 256, 256, 2, 0, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "step 0"),
    ((8, 256, 256, 256, 256, 256, 2, 1, 1e-3, 1.0, 0.999, 1e-8, 0.0, 1.0), "betas"),
    ((8, 256, 256, 256, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 0.0, 0.0, 1.0), "eps"),
    ((8, 256, 256, 256, 256, 256, 2, 1, -1.0, 0.9, 0.999, 1e-8, 0.0, 1.0), "lr"),
    ((8, 256, 256, 256, 256, 256, 2, 1, 1e-3, 0.9, 0.999, 1e-8, -0.1, 1.0), "weight_decay"),
    ((8, 256, 256, 256, 256, 256, 7, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "out_dtype"),
    ((8, 256, None, None, None, None, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "nothing to do"),
    ((8, 256, 256, 256, 256, 0x208, 2, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0), "param_out"),
])
def test_adam_step_validation(lib, args, word):
    """Every rejected argument fails before anything is enqueued (no GPU needed)."""
    assert lib.fno_adam_step(*args, None) == capi.FNO_ERR_INVALID_ARG
    assert word in capi.last_error()


def test_missing_library_raises(tmp_path):
    with pytest.raises(capi.FnoError):
        capi.load(str(tmp_path / "libfno.so"))


@pytest.mark.parametrize("kw,word", [
    ({"step": 0}, "step 0"),
    ({"beta1": 1.5}, "betas (1.5"),
    ({"beta2": -0.5}, "-0.5)"),
    ({"eps": -1.0}, "eps -1"),
    ({"lr": -2.0}, "lr -2"),
    ({"weight_decay": -3.0}, "weight_decay -3"),
    ({"grad_scale": float("inf")}, "grad_scale"),
])
def test_adam_binding_passes_each_argument_in_place(lib, kw, word):
    """The binding's marshalling, checked through the library's validation,
    which runs before anything touches a device (host buffers suffice)."""
    import torch
    t = torch.zeros(16)
    args = dict(step=1, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
                grad_scale=1.0)
    args.update(kw)
    with pytest.raises(capi.FnoError) as e:
        capi.fno_adam_step(t, t.clone(), t.clone(), t.clone(), torch.zeros(16, dtype=torch.bfloat16),
                           stream=0, **args)
    assert e.value.code == capi.FNO_ERR_INVALID_ARG and word in str(e.value)


def test_adam_binding_rejects_a_non_storage_dtype(lib):
    import torch
    t = torch.zeros(8)
    with pytest.raises(ValueError):
        capi.fno_adam_step(t, t, t, t, torch.zeros(8, dtype=torch.float64), 1, 1e-3, stream=0)


_WRAPPERS = {
    "fno_spectral_conv_fwd": ["x", "R", "y", "xhat_save"],
    "fno_spectral_conv_bwd": ["x", "xhat_save", "R", "dy", "dx", "dR"],
    "fno_block_fwd": ["x", "R", "W", "b", "y", "pre_save", "xhat_save"],
    "fno_block_bwd": ["x", "R", "W", "pre_save", "xhat_save", "dy", "dx", "dR", "dW", "db"],
}


@pytest.mark.parametrize("fn,arg", [(f, a) for f, args in _WRAPPERS.items() for a in args])
def test_block_bindings_pass_each_pointer_in_place(lib, fn, arg):
    """A misaligned buffer in one argument of a binding must be reported under
    that argument's name by the library (validation runs before any device
    work, so host buffers suffice)."""
    import torch
    d = capi.block_desc(2, 4, 4, (16, 16), (4, 4))

    def buf(misaligned=False):
        t = torch.zeros(1 << 14)
        return t[1:] if misaligned else t

    kwargs = {name: buf(name == arg) for name in _WRAPPERS[fn]}
    with pytest.raises(capi.FnoError) as e:
        getattr(capi, fn)(d, **kwargs, stream=0)
    assert e.value.code == capi.FNO_ERR_INVALID_ARG
    assert f": {arg} is not 16-byte aligned" in str(e.value)


@pytest.mark.parametrize("which,arg,msg", [
    ("fwd", "a", "a"), ("fwd", "u", "u"), ("fwd", "saves", "saves"),
    ("fwd", "P", "P"), ("fwd", "q1", "q1"), ("fwd", "Q2", "Q2"), ("fwd", "R", "R[l]"),
    ("fwd", "W", "W[l]"), ("fwd", "b", "b[l]"),
    ("bwd", "a", "a"), ("bwd", "saves", "saves"), ("bwd", "du", "du"),
    ("bwd", "gP", "dP"), ("bwd", "gq2", "dq2"),
])
def test_network_bindings_pass_each_pointer_in_place(lib, which, arg, msg):
    import torch
    d = capi.net_desc(2, (16, 16), (4, 4), 3, 8, hidden=16, n_layers=2)

    def buf(misaligned=False):
        t = torch.zeros(1 << 14)
        return t[1:] if misaligned else t

    keys = ("P", "p", "Q1", "q1", "Q2", "q2")
    params = {k: buf(arg == k) for k in keys}
    params.update({k: [buf(arg == k), buf()] for k in ("R", "W", "b")})
    with pytest.raises(capi.FnoError) as e:
        if which == "fwd":
            capi.fno_forward(d, buf(arg == "a"), capi.make_params(params), buf(arg == "u"),
                             buf(arg == "saves"), stream=0)
        else:
            grads = {k: buf(arg == "g" + k) for k in keys}
            grads.update({k: [buf(), buf()] for k in ("R", "W", "b")})
            capi.fno_backward(d, buf(arg == "a"), capi.make_params(params), buf(arg == "saves"),
                              buf(arg == "du"), capi.make_grads(grads), stream=0)
    assert e.value.code == capi.FNO_ERR_INVALID_ARG
    assert f": {msg} is not 16-byte aligned" in str(e.value)


def test_factorised_forward_validation(lib):
    d = capi.block_desc(2, 4, 4, (16, 16), (4, 4))
    need = capi.fno_workspace_size(d, capi.FNO_OP_BLOCK_FWD)
    f = lib.fno_block_fwd_cp
    ok = dict(x=256, lam=256, A=256, B=256, C=256, W=256, b=256, y=256)

    def call(rank, **kw):
        a = dict(ok, **kw)
        return f(ctypes.byref(d), rank, a["x"], a["lam"], a["A"], a["B"], a["C"], a["W"], a["b"],
                 a["y"], None, None, 256, need, None)
    assert call(0) == capi.FNO_ERR_INVALID_ARG and "rank" in capi.last_error()
    assert call(capi.FNO_MAX_CP_RANK + 1) == capi.FNO_ERR_UNSUPPORTED
    for name in ("lam", "A", "B", "C"):
        assert call(4, **{name: None}) == capi.FNO_ERR_INVALID_ARG
        assert name in capi.last_error()
        assert call(4, **{name: 0x1008}) == capi.FNO_ERR_INVALID_ARG
    g = lib.fno_spectral_conv_fwd_cp
    assert g(ctypes.byref(d), 4, 256, 256, 256, 256, 256, 256, None, 256, 1,
             None) == capi.FNO_ERR_WORKSPACE


def test_backward_ready_validation(lib):
    d = capi.net_desc(2, (16, 16), (4, 4), 3, 8, 16, 1, 2)
    need = capi.fno_net_workspace_size(d, capi.FNO_OP_NET_BWD)
    params, grads = capi.Params(), capi.Grads()
    evs = (ctypes.c_void_p * 4)(*([0x100] * 4))
    f = lib.fno_backward_ready
    # wrong count, NULL array with a count, and a NULL event are refused up front
    assert f(ctypes.byref(d), 256, ctypes.byref(params), 256, 256, ctypes.byref(grads), 256, need,
             None, evs, 3) == capi.FNO_ERR_INVALID_ARG
    assert "n_layers + 2" in capi.last_error()
    assert f(ctypes.byref(d), 256, ctypes.byref(params), 256, 256, ctypes.byref(grads), 256, need,
             None, None, 4) == capi.FNO_ERR_INVALID_ARG
    evs[2] = None
    assert f(ctypes.byref(d), 256, ctypes.byref(params), 256, 256, ctypes.byref(grads), 256, need,
             None, evs, 4) == capi.FNO_ERR_INVALID_ARG
    assert "ready[2]" in capi.last_error()


def test_wait_limit_rejects_negative_values(lib):
    assert lib.fno_set_wait_limit(-1) == capi.FNO_ERR_INVALID_ARG
    assert "wait limit" in capi.last_error()


def test_factorised_backward_validation(lib):
    d = capi.block_desc(2, 4, 4, (16, 16), (4, 4))
    need = capi.fno_workspace_size(d, capi.FNO_OP_BLOCK_BWD_CP)
    assert need > capi.fno_workspace_size(d, capi.FNO_OP_BLOCK_BWD)
    assert capi.fno_workspace_size(d, capi.FNO_OP_SPECTRAL_BWD_CP) > 0
    f = lib.fno_block_bwd_cp
    ok = dict(x=256, lam=256, A=256, B=256, C=256, W=256, pre=256, dy=256, dx=256, dlam=256,
              dA=256, dB=256, dC=256, dW=256, db=256)

    def call(rank, ws=need, **kw):
        a = dict(ok, **kw)
        return f(ctypes.byref(d), rank, a["x"], a["lam"], a["A"], a["B"], a["C"], a["W"],
                 a["pre"], None, a["dy"], a["dx"], a["dlam"], a["dA"], a["dB"], a["dC"], a["dW"],
                 a["db"], 256, ws, None)
    assert call(0) == capi.FNO_ERR_INVALID_ARG
    assert call(capi.FNO_MAX_CP_RANK + 1) == capi.FNO_ERR_UNSUPPORTED
    for name in ("dlam", "dA", "dB", "dC", "dW", "db", "dx", "dy"):
        assert call(4, **{name: None}) == capi.FNO_ERR_INVALID_ARG
        assert name in capi.last_error()
    assert call(4, ws=need - 1) == capi.FNO_ERR_WORKSPACE


def _header_arities():
    """Number of parameters of every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(fno_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(lib):
    """Every ctypes signature declares exactly the header's parameter count, so
    no argument (the stream last of all) is ever passed with default conversion."""
    arities = _header_arities()
    assert set(arities) == set(capi.EXPORTED)
    for name, n in arities.items():
        assert len(getattr(lib, name).argtypes) == n, name
