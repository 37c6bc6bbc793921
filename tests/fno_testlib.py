"""Helpers shared by the GPU parity tests: device upload, CUDA-path calls through
the C ABI, oracle calls and the relative-L2 comparison."""

from __future__ import annotations

import numpy as np

import oracle as O
from fourier_neural_spectral_fno_b200 import capi

TOL = {"f32": 1e-5, "f16": 1e-2, "bf16": 1e-2}


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def dev(a, dtype: str = "f32"):
    """Upload a float64 array (already rounded to ``dtype``) as a CUDA tensor."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(torch_dtype(dtype))


def dev_complex(z, dtype: str = "f32"):
    """Complex array -> [..., 2] real CUDA tensor in the storage dtype."""
    z = np.asarray(z)
    return dev(np.stack([z.real, z.imag], axis=-1), dtype)


def host(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def host_complex(t) -> np.ndarray:
    a = host(t)
    return a[..., 0] + 1j * a[..., 1]


def empty(shape, dtype: str = "f32"):
    import torch
    return torch.empty(tuple(shape), dtype=torch_dtype(dtype), device="cuda")


def rel_l2(got, ref) -> float:
    got = np.asarray(got)
    ref = np.asarray(ref)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / (den if den > 0 else 1.0))


def assert_close(got, ref, tol, what=""):
    err = rel_l2(got, ref)
    assert np.all(np.isfinite(np.asarray(got))), f"{what}: non-finite values"
    assert err <= tol, f"{what}: relative L2 error {err:.3e} > {tol:.1e}"
    return err


def flags_of(tanh=False, no_act=False) -> int:
    return (capi.FNO_TANH_PREACT if tanh else 0) | (capi.FNO_NO_ACT if no_act else 0)


def oracle_flags(flags: int) -> int:
    return (O.TANH_PREACT if flags & capi.FNO_TANH_PREACT else 0) | \
        (O.NO_ACT if flags & capi.FNO_NO_ACT else 0)


def params_to_device(params, dtype):
    out = {}
    for key, val in params.items():
        if isinstance(val, list):
            out[key] = [dev_complex(v, dtype) if np.iscomplexobj(v) else dev(v, dtype) for v in val]
        else:
            out[key] = dev(val, dtype)
    return out


def grads_like(params):
    import torch
    out = {}
    for key, val in params.items():
        if isinstance(val, list):
            out[key] = [torch.empty(v.shape + ((2,) if np.iscomplexobj(v) else ()),
                                    dtype=torch.float32, device="cuda") for v in val]
        else:
            out[key] = torch.empty(np.shape(val), dtype=torch.float32, device="cuda")
    return out
