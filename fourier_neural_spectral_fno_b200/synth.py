"""Seeded synthetic inputs and parameters for the FNO workloads.

This module only draws numbers: Gaussian random fields, coordinate grids,
parameter initialisation and storage-dtype rounding.  It holds none of the
block's arithmetic, and it is the one module that both the CUDA path (through
the tests and the benchmark) and the CPU oracle receive their inputs from.

The workloads stand in for the pages' data sets, which are not available:
the magnetotelluric resistivity models of "Efficient multi-GPU distributed
training strategies for neural operator networks: Application to
magnetotelluric forward modeling" (key methods), and the 512^3 volumes of
"Model-Parallel Fourier Neural Operators as Learned Surrogates for Large-Scale
Parametric PDEs" (main findings).  A log-resistivity model is represented by a
standardised Gaussian random field with power spectrum ``(1 + |k|^2)^-2``,
concatenated with its coordinate grids.

Seeds (``numpy.random.default_rng``): inputs 0, weights 1, target 2,
cotangent 3.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

SEED_INPUT, SEED_WEIGHTS, SEED_TARGET, SEED_COTANGENT = 0, 1, 2, 3

DTYPES = ("f32", "f16", "bf16")


# --------------------------------------------------------------------------
# storage rounding (round to nearest even, then back to float64)
# --------------------------------------------------------------------------

def _round_bf16(a: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    out = (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return out.astype(np.float64)


def quantize(a, dtype: str) -> np.ndarray:
    """Round ``a`` to the storage dtype and return it as float64."""
    a = np.asarray(a, dtype=np.float64)
    if dtype == "f32":
        return a.astype(np.float32).astype(np.float64)
    if dtype == "f16":
        return a.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        return _round_bf16(a)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# fields
# --------------------------------------------------------------------------

def _wavenumber_norm2(grid: Sequence[int]) -> np.ndarray:
    """|k|^2 on the half spectrum, with signed integer wavenumbers."""
    d = len(grid)
    axes = []
    for j, n in enumerate(grid):
        if j == d - 1:
            axes.append(np.arange(n // 2 + 1, dtype=np.float64))
        else:
            k = np.arange(n, dtype=np.float64)
            axes.append(np.where(k <= n // 2, k, k - n))
    mesh = np.meshgrid(*axes, indexing="ij")
    return sum(m * m for m in mesh)


def gaussian_random_field(rng: np.random.Generator, count: int,
                          grid: Sequence[int], lowpass: Optional[float] = None) -> np.ndarray:
    """``count`` standardised fields with power spectrum ``(1 + |k|^2)^-2``.

    Complex white noise on the half spectrum is scaled by the amplitude
    ``(1 + |k|^2)^-1`` (optionally times ``exp(-|k|^2 / (2 lowpass^2))``),
    brought to the grid with NumPy's inverse real FFT, and each field is
    shifted and scaled to mean 0 and standard deviation 1.
    """
    grid = tuple(int(n) for n in grid)
    k2 = _wavenumber_norm2(grid)
    amp = 1.0 / (1.0 + k2)
    if lowpass is not None:
        amp = amp * np.exp(-k2 / (2.0 * lowpass * lowpass))
    out = np.empty((count,) + grid, dtype=np.float64)
    axes = tuple(range(len(grid)))
    for i in range(count):
        noise = rng.standard_normal(k2.shape) + 1j * rng.standard_normal(k2.shape)
        f = np.fft.irfftn(noise * amp, s=grid, axes=axes)
        f -= f.mean()
        f /= f.std()
        out[i] = f
    return out


def coordinate_grids(grid: Sequence[int]) -> np.ndarray:
    """``[d, *grid]``: channel j holds ``linspace(0, 1, N_j)`` along axis j."""
    lin = [np.linspace(0.0, 1.0, int(n)) for n in grid]
    return np.stack(np.meshgrid(*lin, indexing="ij"), axis=0)


def resistivity_input(rng: np.random.Generator, batch: int, grid: Sequence[int]) -> np.ndarray:
    """``[B, 1 + d, *grid]``: a log-resistivity field and its coordinates."""
    field = gaussian_random_field(rng, batch, grid)
    coords = coordinate_grids(grid)
    out = np.empty((batch, 1 + len(grid)) + tuple(grid), dtype=np.float64)
    out[:, 0] = field
    out[:, 1:] = coords[None]
    return out


# --------------------------------------------------------------------------
# parameters
# --------------------------------------------------------------------------

def _uniform(rng, shape, bound):
    return rng.uniform(-bound, bound, size=shape)


def spectral_weights(rng: np.random.Generator, cin: int, cout: int, n_modes: int) -> np.ndarray:
    """``R[i, o, k]`` complex: real and imaginary parts ~ U(0, 1) / (cin * cout)."""
    scale = 1.0 / (cin * cout)
    re = rng.uniform(0.0, 1.0, size=(cin, cout, n_modes)) * scale
    im = rng.uniform(0.0, 1.0, size=(cin, cout, n_modes)) * scale
    return re + 1j * im


def block_params(rng: np.random.Generator, cin: int, cout: int, n_modes: int,
                 bias: bool = False) -> Dict[str, np.ndarray]:
    """One block: ``R``, ``W ~ U(+-1/sqrt(cin))`` and ``b`` (0 unless ``bias``)."""
    r = spectral_weights(rng, cin, cout, n_modes)
    w = _uniform(rng, (cout, cin), 1.0 / np.sqrt(cin))
    b = _uniform(rng, (cout,), 1.0 / np.sqrt(cin)) if bias else np.zeros(cout)
    return {"R": r, "W": w, "b": b}


def network_params(rng: np.random.Generator, in_ch: int, width: int, hidden: int,
                   out_ch: int, n_layers: int, n_modes: int) -> Dict[str, object]:
    """Lift ``P, p``; per block ``R, W, b``; projection ``Q1, q1, Q2, q2``.

    Lift and projection weights and biases ~ U(+-1/sqrt(fan_in)).
    """
    params: Dict[str, object] = {
        "P": _uniform(rng, (width, in_ch), 1.0 / np.sqrt(in_ch)),
        "p": _uniform(rng, (width,), 1.0 / np.sqrt(in_ch)),
        "R": [], "W": [], "b": [],
    }
    for _ in range(n_layers):
        bp = block_params(rng, width, width, n_modes)
        params["R"].append(bp["R"])
        params["W"].append(bp["W"])
        params["b"].append(bp["b"])
    params["Q1"] = _uniform(rng, (hidden, width), 1.0 / np.sqrt(width))
    params["q1"] = _uniform(rng, (hidden,), 1.0 / np.sqrt(width))
    params["Q2"] = _uniform(rng, (out_ch, hidden), 1.0 / np.sqrt(hidden))
    params["q2"] = _uniform(rng, (out_ch,), 1.0 / np.sqrt(hidden))
    return params


def quantize_params(params: Dict[str, object], dtype: str) -> Dict[str, object]:
    """Round every parameter (real and imaginary parts alike) to ``dtype``."""
    out: Dict[str, object] = {}
    for key, val in params.items():
        if isinstance(val, list):
            out[key] = [quantize_complex(v, dtype) if np.iscomplexobj(v) else quantize(v, dtype)
                        for v in val]
        elif np.iscomplexobj(val):
            out[key] = quantize_complex(val, dtype)
        else:
            out[key] = quantize(val, dtype)
    return out


def quantize_complex(z, dtype: str) -> np.ndarray:
    z = np.asarray(z)
    return quantize(z.real, dtype) + 1j * quantize(z.imag, dtype)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "block" or "network"
    dtype: str
    batch: int
    grid: Tuple[int, ...]
    modes: Tuple[int, ...]
    width: int
    in_ch: int = 0            # network input channels (field + coordinates)
    hidden: int = 128
    out_ch: int = 1
    n_layers: int = 4
    tanh: bool = False
    backward: bool = False
    description: str = ""

    @property
    def ndim(self) -> int:
        return len(self.grid)

    @property
    def points(self) -> int:
        return int(np.prod(self.grid))


WORKLOADS: Dict[str, Workload] = {
    "block2d_f32_b4_w20_64sq_m12": Workload(
        "block2d_f32_b4_w20_64sq_m12", "block", "f32", 4, (64, 64), (12, 12), 20,
        description="single 2D spectral block, fp32, x ~ N(0,1), forward"),
    "fno2d_f32_b16_w32_256sq_m16": Workload(
        "fno2d_f32_b16_w32_256sq_m16", "network", "f32", 16, (256, 256), (16, 16), 32,
        in_ch=3, description="2D FNO forward: lift 3->32, 4 blocks, projection 32->128->1"),
    "block2d_f16tanh_b8_w64_512sq_m32": Workload(
        "block2d_f16tanh_b8_w64_512sq_m32", "block", "f16", 8, (512, 512), (32, 32), 64,
        tanh=True, backward=True,
        description="2D block, fp16 storage, tanh pre-activation, forward + backward"),
    "fno3d_f32_b2_w20_128cube_m8": Workload(
        "fno3d_f32_b2_w20_128cube_m8", "network", "f32", 2, (128, 128, 128), (8, 8, 8), 20,
        in_ch=4, description="3D FNO forward: lift 4->20, 4 blocks, projection 20->128->1"),
    "fno2d_bf16_train_b32_w64_256sq_m24": Workload(
        "fno2d_bf16_train_b32_w64_256sq_m24", "network", "bf16", 32, (256, 256), (24, 24), 64,
        in_ch=3, backward=True,
        description="2D FNO training step, bf16 storage, MSE against a smoothed field"),
}

WORKLOAD_ORDER: List[str] = list(WORKLOADS)


def make_block_inputs(wl: Workload, batch: Optional[int] = None, grid=None,
                      bias: bool = False) -> Dict[str, np.ndarray]:
    """Block-workload inputs, already rounded to the storage dtype (float64)."""
    batch = wl.batch if batch is None else batch
    grid = wl.grid if grid is None else tuple(grid)
    rng_in = np.random.default_rng(SEED_INPUT)
    if wl.dtype == "f32":
        x = rng_in.standard_normal((batch, wl.width) + grid)
    else:
        x = gaussian_random_field(rng_in, batch * wl.width, grid).reshape(
            (batch, wl.width) + grid)
    n_modes = _num_kept(grid, wl.modes)
    p = block_params(np.random.default_rng(SEED_WEIGHTS), wl.width, wl.width, n_modes, bias)
    out = {"x": quantize(x, wl.dtype), "R": quantize_complex(p["R"], wl.dtype),
           "W": quantize(p["W"], wl.dtype), "b": quantize(p["b"], wl.dtype)}
    if wl.backward:
        dy = np.random.default_rng(SEED_COTANGENT).standard_normal((batch, wl.width) + grid)
        out["dy"] = quantize(dy, wl.dtype)
    return out


def make_network_inputs(wl: Workload, batch: Optional[int] = None, grid=None) -> Dict[str, object]:
    """Network-workload input ``a``, parameters and (training) target."""
    batch = wl.batch if batch is None else batch
    grid = wl.grid if grid is None else tuple(grid)
    a = resistivity_input(np.random.default_rng(SEED_INPUT), batch, grid)
    n_modes = _num_kept(grid, wl.modes)
    params = network_params(np.random.default_rng(SEED_WEIGHTS), wl.in_ch, wl.width,
                            wl.hidden, wl.out_ch, wl.n_layers, n_modes)
    out: Dict[str, object] = {"a": quantize(a, wl.dtype),
                              "params": quantize_params(params, wl.dtype)}
    if wl.backward:
        t = gaussian_random_field(np.random.default_rng(SEED_TARGET), batch * wl.out_ch,
                                  grid, lowpass=8.0)
        out["target"] = quantize(t.reshape((batch, wl.out_ch) + grid), wl.dtype)
    return out


def _num_kept(grid, modes) -> int:
    """|K| = m_last * prod_{j<d-1} 2 m_j (pure counting)."""
    n = int(modes[-1])
    for m in modes[:-1]:
        n *= 2 * int(m)
    return n
