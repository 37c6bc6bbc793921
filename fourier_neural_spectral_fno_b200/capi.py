"""Thin ctypes binding of ``libfno.so`` (the C ABI declared in ``include/fno.h``).

Argument marshalling only: every function here turns torch tensors into device
pointers (plus the current CUDA stream) and calls the C entry point of the
same name; all arithmetic runs in the library's CUDA kernels.  Workspaces and
outputs are allocated with torch when the caller does not pass them.

Importing this module does not touch the GPU.  The library is loaded on the
first call; if ``libfno.so`` is missing the call raises -- there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfno.so")

FNO_OK = 0
FNO_ERR_INVALID_ARG = -1
FNO_ERR_UNSUPPORTED = -2
FNO_ERR_WORKSPACE = -3
FNO_ERR_CUDA = -4
FNO_ERR_TIMEOUT = -5

FNO_F32, FNO_F16, FNO_BF16 = 0, 1, 2
DTYPE_CODE = {"f32": FNO_F32, "f16": FNO_F16, "bf16": FNO_BF16}

FNO_TANH_PREACT = 1
FNO_NO_ACT = 2

FNO_OP_SPECTRAL_FWD, FNO_OP_SPECTRAL_BWD, FNO_OP_BLOCK_FWD, FNO_OP_BLOCK_BWD = 0, 1, 2, 3
FNO_OP_NET_FWD, FNO_OP_NET_BWD = 4, 5
FNO_OP_SPECTRAL_BWD_CP, FNO_OP_BLOCK_BWD_CP = 6, 7

FNO_MAX_DIMS = 3
FNO_MAX_LAYERS = 16

# every symbol include/fno.h declares
EXPORTED = (
    "fno_last_error", "fno_version", "fno_last_launch_count", "fno_workspace_size",
    "fno_net_workspace_size", "fno_net_saves_size", "fno_spectral_conv_fwd",
    "fno_spectral_conv_bwd", "fno_block_fwd", "fno_block_bwd", "fno_forward", "fno_backward",
    "fno_mse", "fno_profile_enable", "fno_profile_read", "fno_set_tensor_cores",
    "fno_device_error", "fno_spectral_conv_fwd_noalloc", "fno_adam_step",
    "fno_backward_ready", "fno_spectral_conv_fwd_cp", "fno_block_fwd_cp", "fno_set_wait_limit",
    "fno_spectral_conv_bwd_cp", "fno_block_bwd_cp",
)

FNO_MAX_CP_RANK = 32
FNO_NOALLOC_SCRATCH_BYTES = 32 << 20


class FnoError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"fno error {code}: {msg}")
        self.code = code


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


class BlockDesc(ctypes.Structure):
    _fields_ = [
        ("ndim", ctypes.c_int), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint),
        ("cin", ctypes.c_int), ("cout", ctypes.c_int), ("batch", ctypes.c_int64),
        ("grid", ctypes.c_int64 * FNO_MAX_DIMS), ("modes", ctypes.c_int * FNO_MAX_DIMS),
    ]


class NetDesc(ctypes.Structure):
    _fields_ = [
        ("ndim", ctypes.c_int), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint),
        ("in_channels", ctypes.c_int), ("width", ctypes.c_int), ("hidden", ctypes.c_int),
        ("out_channels", ctypes.c_int), ("n_layers", ctypes.c_int), ("batch", ctypes.c_int64),
        ("grid", ctypes.c_int64 * FNO_MAX_DIMS), ("modes", ctypes.c_int * FNO_MAX_DIMS),
    ]


_PARR = ctypes.c_void_p * FNO_MAX_LAYERS


class Params(ctypes.Structure):
    _fields_ = [("P", ctypes.c_void_p), ("p", ctypes.c_void_p), ("R", _PARR), ("W", _PARR),
                ("b", _PARR), ("Q1", ctypes.c_void_p), ("q1", ctypes.c_void_p),
                ("Q2", ctypes.c_void_p), ("q2", ctypes.c_void_p)]


class Grads(Params):
    pass


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load ``libfno.so`` once and declare the C signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise FnoError(FNO_ERR_CUDA, f"{path} is missing; build it with "
                       "`python -m fourier_neural_spectral_fno_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    bd, nd = ctypes.POINTER(BlockDesc), ctypes.POINTER(NetDesc)
    sig = {
        "fno_last_error": (ctypes.c_char_p, []),
        "fno_version": (ctypes.c_char_p, []),
        "fno_last_launch_count": (i, []),
        "fno_workspace_size": (sz, [bd, i]),
        "fno_net_workspace_size": (sz, [nd, i]),
        "fno_net_saves_size": (sz, [nd]),
        "fno_spectral_conv_fwd": (i, [bd, vp, vp, vp, vp, vp, sz, vp]),
        "fno_spectral_conv_bwd": (i, [bd, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fno_block_fwd": (i, [bd, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fno_block_bwd": (i, [bd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fno_forward": (i, [nd, vp, ctypes.POINTER(Params), vp, vp, vp, sz, vp]),
        "fno_backward": (i, [nd, vp, ctypes.POINTER(Params), vp, vp, ctypes.POINTER(Grads), vp,
                             sz, vp]),
        "fno_backward_ready": (i, [nd, vp, ctypes.POINTER(Params), vp, vp,
                                   ctypes.POINTER(Grads), vp, sz, vp,
                                   ctypes.POINTER(ctypes.c_void_p), i]),
        "fno_mse": (i, [ctypes.c_int64, i, vp, vp, vp, vp, vp]),
        "fno_profile_enable": (i, [i]),
        "fno_set_tensor_cores": (i, [i]),
        "fno_spectral_conv_fwd_noalloc": (i, [bd, vp, vp, vp, vp, vp]),
        "fno_spectral_conv_fwd_cp": (i, [bd, i, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fno_block_fwd_cp": (i, [bd, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "fno_spectral_conv_bwd_cp": (i, [bd, i] + [vp] * 13 + [sz, vp]),
        "fno_block_bwd_cp": (i, [bd, i] + [vp] * 17 + [sz, vp]),
        "fno_device_error": (i, [i]),
        "fno_set_wait_limit": (i, [i]),
        "fno_profile_read": (i, [ctypes.POINTER(KernelStat), i]),
        "fno_adam_step": (i, [ctypes.c_int64, vp, vp, vp, vp, vp, i, i, ctypes.c_float,
                              ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                              ctypes.c_float, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def last_error() -> str:
    return load().fno_last_error().decode()


def last_launch_count() -> int:
    return load().fno_last_launch_count()


def _check(rc: int) -> None:
    if rc != FNO_OK:
        raise FnoError(rc, last_error())


# --------------------------------------------------------------------------
# descriptors
# --------------------------------------------------------------------------

def block_desc(batch: int, cin: int, cout: int, grid: Sequence[int], modes: Sequence[int],
               dtype: str = "f32", flags: int = 0) -> BlockDesc:
    d = BlockDesc()
    d.ndim = len(grid)
    d.dtype = DTYPE_CODE[dtype]
    d.flags = flags
    d.cin, d.cout, d.batch = cin, cout, batch
    for j, (n, m) in enumerate(zip(grid, modes)):
        d.grid[j], d.modes[j] = int(n), int(m)
    return d


def net_desc(batch: int, grid: Sequence[int], modes: Sequence[int], in_channels: int, width: int,
             hidden: int = 128, out_channels: int = 1, n_layers: int = 4, dtype: str = "f32",
             flags: int = 0) -> NetDesc:
    d = NetDesc()
    d.ndim = len(grid)
    d.dtype = DTYPE_CODE[dtype]
    d.flags = flags
    d.in_channels, d.width, d.hidden = in_channels, width, hidden
    d.out_channels, d.n_layers, d.batch = out_channels, n_layers, batch
    for j, (n, m) in enumerate(zip(grid, modes)):
        d.grid[j], d.modes[j] = int(n), int(m)
    return d


def num_modes(grid: Sequence[int], modes: Sequence[int]) -> int:
    k = int(modes[-1])
    for m in modes[:-1]:
        k *= 2 * int(m)
    return k


# --------------------------------------------------------------------------
# tensor marshalling
# --------------------------------------------------------------------------

def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _workspace(nbytes: int, device, ws):
    import torch
    if ws is not None:
        return ws, ws.numel() * ws.element_size()
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device), max(nbytes, 256)


def fno_workspace_size(desc: BlockDesc, op: int) -> int:
    n = load().fno_workspace_size(ctypes.byref(desc), op)
    if n == 0:
        raise FnoError(FNO_ERR_INVALID_ARG, last_error())
    return n


def fno_net_workspace_size(desc: NetDesc, op: int) -> int:
    n = load().fno_net_workspace_size(ctypes.byref(desc), op)
    if n == 0:
        raise FnoError(FNO_ERR_INVALID_ARG, last_error())
    return n


def fno_net_saves_size(desc: NetDesc) -> int:
    n = load().fno_net_saves_size(ctypes.byref(desc))
    if n == 0:
        raise FnoError(FNO_ERR_INVALID_ARG, last_error())
    return n


def fno_spectral_conv_fwd(desc, x, R, y, xhat_save=None, ws=None, stream=None):
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_SPECTRAL_FWD), x.device, ws)
    _check(load().fno_spectral_conv_fwd(ctypes.byref(desc), _ptr(x), _ptr(R), _ptr(y),
                                        _ptr(xhat_save), _ptr(ws), nb, _stream(stream)))
    return y


def fno_spectral_conv_bwd(desc, x, xhat_save, R, dy, dx, dR, ws=None, stream=None):
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_SPECTRAL_BWD), x.device, ws)
    _check(load().fno_spectral_conv_bwd(ctypes.byref(desc), _ptr(x), _ptr(xhat_save), _ptr(R),
                                        _ptr(dy), _ptr(dx), _ptr(dR), _ptr(ws), nb,
                                        _stream(stream)))
    return dx, dR


def fno_block_fwd(desc, x, R, W, b, y, pre_save=None, xhat_save=None, ws=None, stream=None):
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_BLOCK_FWD), x.device, ws)
    _check(load().fno_block_fwd(ctypes.byref(desc), _ptr(x), _ptr(R), _ptr(W), _ptr(b), _ptr(y),
                                _ptr(pre_save), _ptr(xhat_save), _ptr(ws), nb, _stream(stream)))
    return y


def fno_spectral_conv_fwd_cp(desc, rank, x, lam, A, B, C, y, xhat_save=None, ws=None,
                             stream=None):
    """Spectral forward with CP-factorised weights (factors [..][rank][2])."""
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_SPECTRAL_FWD), x.device, ws)
    _check(load().fno_spectral_conv_fwd_cp(ctypes.byref(desc), int(rank), _ptr(x), _ptr(lam),
                                           _ptr(A), _ptr(B), _ptr(C), _ptr(y), _ptr(xhat_save),
                                           _ptr(ws), nb, _stream(stream)))
    return y


def fno_block_fwd_cp(desc, rank, x, lam, A, B, C, W, b, y, pre_save=None, xhat_save=None,
                     ws=None, stream=None):
    """Block forward with CP-factorised weights (factors [..][rank][2])."""
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_BLOCK_FWD), x.device, ws)
    _check(load().fno_block_fwd_cp(ctypes.byref(desc), int(rank), _ptr(x), _ptr(lam), _ptr(A),
                                   _ptr(B), _ptr(C), _ptr(W), _ptr(b), _ptr(y), _ptr(pre_save),
                                   _ptr(xhat_save), _ptr(ws), nb, _stream(stream)))
    return y


def fno_spectral_conv_bwd_cp(desc, rank, x, lam, A, B, C, xhat_save, dy, dx, dlam, dA, dB, dC,
                             ws=None, stream=None):
    """Adjoint of :func:`fno_spectral_conv_fwd_cp`: dx and the factor gradients."""
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_SPECTRAL_BWD_CP), x.device, ws)
    _check(load().fno_spectral_conv_bwd_cp(ctypes.byref(desc), int(rank), _ptr(x), _ptr(lam),
                                           _ptr(A), _ptr(B), _ptr(C), _ptr(xhat_save), _ptr(dy),
                                           _ptr(dx), _ptr(dlam), _ptr(dA), _ptr(dB), _ptr(dC),
                                           _ptr(ws), nb, _stream(stream)))
    return dx, dlam, dA, dB, dC


def fno_block_bwd_cp(desc, rank, x, lam, A, B, C, W, pre_save, xhat_save, dy, dx, dlam, dA, dB,
                     dC, dW, db, ws=None, stream=None):
    """Adjoint of :func:`fno_block_fwd_cp`: dx, the factor gradients, dW and db."""
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_BLOCK_BWD_CP), x.device, ws)
    _check(load().fno_block_bwd_cp(ctypes.byref(desc), int(rank), _ptr(x), _ptr(lam), _ptr(A),
                                   _ptr(B), _ptr(C), _ptr(W), _ptr(pre_save), _ptr(xhat_save),
                                   _ptr(dy), _ptr(dx), _ptr(dlam), _ptr(dA), _ptr(dB), _ptr(dC),
                                   _ptr(dW), _ptr(db), _ptr(ws), nb, _stream(stream)))
    return dx, dlam, dA, dB, dC, dW, db


def fno_block_bwd(desc, x, R, W, pre_save, xhat_save, dy, dx, dR, dW, db, ws=None, stream=None):
    ws, nb = _workspace(fno_workspace_size(desc, FNO_OP_BLOCK_BWD), x.device, ws)
    _check(load().fno_block_bwd(ctypes.byref(desc), _ptr(x), _ptr(R), _ptr(W), _ptr(pre_save),
                                _ptr(xhat_save), _ptr(dy), _ptr(dx), _ptr(dR), _ptr(dW), _ptr(db),
                                _ptr(ws), nb, _stream(stream)))
    return dx, dR, dW, db


def make_params(tensors: Dict[str, object]) -> Params:
    """``Params`` from a dict of device tensors (``R``, ``W``, ``b`` are lists)."""
    p = Params()
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        setattr(p, key, _ptr(tensors[key]))
    for key in ("R", "W", "b"):
        arr = getattr(p, key)
        for l, t in enumerate(tensors[key]):
            arr[l] = _ptr(t)
    return p


def make_grads(tensors: Dict[str, object]) -> Grads:
    g = Grads()
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        setattr(g, key, _ptr(tensors[key]))
    for key in ("R", "W", "b"):
        arr = getattr(g, key)
        for l, t in enumerate(tensors[key]):
            arr[l] = _ptr(t)
    return g


def fno_forward(desc, a, params: Params, u, saves=None, ws=None, stream=None):
    ws, nb = _workspace(fno_net_workspace_size(desc, FNO_OP_NET_FWD), a.device, ws)
    _check(load().fno_forward(ctypes.byref(desc), _ptr(a), ctypes.byref(params), _ptr(u),
                              _ptr(saves), _ptr(ws), nb, _stream(stream)))
    return u


def fno_backward(desc, a, params: Params, saves, du, grads: Grads, ws=None, stream=None,
                 ready=None):
    """``ready``: optional list of n_layers + 2 ``torch.cuda.Event`` that the
    backward records as each gradient group becomes final (fno_backward_ready):
    the projection's, then the layers' from the last to the first, then the lift's."""
    ws, nb = _workspace(fno_net_workspace_size(desc, FNO_OP_NET_BWD), a.device, ws)
    if ready is None:
        _check(load().fno_backward(ctypes.byref(desc), _ptr(a), ctypes.byref(params), _ptr(saves),
                                   _ptr(du), ctypes.byref(grads), _ptr(ws), nb, _stream(stream)))
        return
    handles = []
    for ev in ready:
        if ev.cuda_event == 0:      # torch creates the event lazily, on its first record
            ev.record()
        handles.append(ev.cuda_event)
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _check(load().fno_backward_ready(ctypes.byref(desc), _ptr(a), ctypes.byref(params),
                                     _ptr(saves), _ptr(du), ctypes.byref(grads), _ptr(ws), nb,
                                     _stream(stream), arr, len(handles)))
    return grads


def fno_mse(u, target, loss, du=None, dtype: str = "f32", stream=None):
    _check(load().fno_mse(u.numel(), DTYPE_CODE[dtype], _ptr(u), _ptr(target), _ptr(loss), _ptr(du),
                          _stream(stream)))
    return loss


def fno_profile_enable(on: bool = True) -> None:
    _check(load().fno_profile_enable(1 if on else 0))


def fno_profile_read(max_kernels: int = 64) -> Dict[str, Dict[str, float]]:
    """Per-kernel launches and summed device time (ms) since the last enable."""
    arr = (KernelStat * max_kernels)()
    n = load().fno_profile_read(arr, max_kernels)
    if n < 0:
        raise FnoError(n, last_error())
    return {arr[i].name.decode(): {"launches": arr[i].launches, "total_ms": arr[i].total_ms}
            for i in range(n)}


def fno_set_tensor_cores(mode) -> int:
    """Kernel selection: 1 / True = the default kernels (per shape the faster
    design as measured: the streaming pruned-FFT transform, mixing (tcgen05
    for bfloat16 weights with 64 output channels) and pruned slab-axis inverse
    on the CUDA cores, tcgen05 TMA pipelines for the epilogue and projection),
    4 = the default with the clustered FFT transform, 3 =
    tcgen05 TMA pipelines throughout (dense DFT-matrix transform), 2 = tcgen05
    kernels without the pipelines, 0 / False = the CUDA-core kernels.  Returns
    the previous setting."""
    m = int(mode)
    if m not in (0, 1, 2, 3, 4):
        raise ValueError("kernel mode must be 0, 1, 2, 3 or 4")
    return int(load().fno_set_tensor_cores(m))


def fno_set_wait_limit(spins: int) -> int:
    """Bound every tensor-core pipeline wait to ``spins`` suspended polls
    (default 131072, about two seconds); returns the previous bound.  A test
    hook: 0 makes waits give up after one probe (results then invalid)."""
    prev = int(load().fno_set_wait_limit(int(spins)))
    if prev < 0:
        _check(prev)
    return prev


def fno_device_error(clear: bool = True) -> None:
    """Raise if a bounded device-side wait expired since the last clear."""
    _check(load().fno_device_error(1 if clear else 0))


def fno_spectral_conv_fwd_noalloc(desc, x, R, y, xhat_save=None, stream=None):
    """fno_spectral_conv_fwd with the library's built-in scratch (no workspace)."""
    _check(load().fno_spectral_conv_fwd_noalloc(ctypes.byref(desc), _ptr(x), _ptr(R), _ptr(y),
                                                _ptr(xhat_save), _stream(stream)))
    return y


def _dtype_code_of(t) -> int:
    import torch
    codes = {torch.float32: FNO_F32, torch.float16: FNO_F16, torch.bfloat16: FNO_BF16}
    if t.dtype not in codes:
        raise ValueError(f"param_out dtype {t.dtype} is not a storage dtype")
    return codes[t.dtype]


def fno_adam_step(theta, m, v, grad, param_out, step: int, lr: float, beta1: float = 0.9,
                  beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                  grad_scale: float = 1.0, stream=None):
    """One Adam step on the float32 master ``theta`` (with moments ``m``, ``v``)
    fused with the copy into ``param_out`` (its torch dtype is the storage
    dtype).  ``grad=None``: copy only; ``param_out=None``: update only."""
    out_code = _dtype_code_of(param_out) if param_out is not None else FNO_F32
    _check(load().fno_adam_step(theta.numel(), _ptr(theta), _ptr(m), _ptr(v), _ptr(grad),
                                _ptr(param_out), out_code, int(step), float(lr), float(beta1),
                                float(beta2), float(eps), float(weight_decay), float(grad_scale),
                                _stream(stream)))
