"""Per-stage device times of the spectral block for each kernel design.

    python -m fourier_neural_spectral_fno_b200.stage_bench [--steps K] [--out FILE]

For every workload's block shape (batch, width, grid, modes, storage dtype,
flags) the block forward and backward run through the C ABI on each kernel
path of ``fno_set_tensor_cores`` and the library's per-kernel CUDA events
(``fno_profile_enable`` / ``fno_profile_read``) give the mean device time of
every kernel per call.  This is the measurement that chooses between the
truncated transform as a pruned radix-16 FFT on the CUDA cores (path 1) and as
a dense DFT-matrix contraction on the tensor cores (path 3) per stage.
Inputs are seeded synthetic tensors of the workloads' shapes; L2 is flushed
between calls.  Prints a Markdown table (and writes it to ``--out``).
"""

from __future__ import annotations

import argparse

import numpy as np

from . import capi, synth

PATHS = {1: "pruned FFT (CUDA cores)", 3: "DFT matrix (tcgen05)"}


def _time_block(wl, path: int, steps: int):
    import torch
    dt = wl.dtype
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dt]
    flags = capi.FNO_TANH_PREACT if wl.tanh else 0
    C, k = wl.width, capi.num_modes(wl.grid, wl.modes)
    rng = np.random.default_rng(0)
    shape = (wl.batch, C) + tuple(wl.grid)
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).cuda().to(tdt)
    dy = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).cuda().to(tdt)
    r = torch.from_numpy(rng.uniform(0, 1, (C, C, k, 2)).astype(np.float32) / (C * C)).cuda().to(tdt)
    w = torch.from_numpy(rng.uniform(-1, 1, (C, C)).astype(np.float32) / np.sqrt(C)).cuda().to(tdt)
    b = torch.zeros(C, dtype=tdt, device="cuda")
    d = capi.block_desc(wl.batch, C, C, wl.grid, wl.modes, dt, flags)
    y, pre = torch.empty_like(x), torch.empty_like(x)
    xh = torch.empty((wl.batch, C, k, 2), device="cuda")
    dx = torch.empty_like(x)
    dr = torch.empty((C, C, k, 2), device="cuda")
    dw, db = torch.empty((C, C), device="cuda"), torch.empty(C, device="cuda")
    ws = torch.empty(max(capi.fno_workspace_size(d, capi.FNO_OP_BLOCK_FWD),
                         capi.fno_workspace_size(d, capi.FNO_OP_BLOCK_BWD)),
                     dtype=torch.uint8, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    prev = capi.fno_set_tensor_cores(path)
    try:
        def call():
            capi.fno_block_fwd(d, x, r, w, b, y, pre, xh, ws)
            capi.fno_block_bwd(d, x, r, w, pre, xh, dy, dx, dr, dw, db, ws)
        for _ in range(2):
            call()
        torch.cuda.synchronize()
        capi.fno_profile_enable(True)
        for i in range(steps):
            flush.fill_(i & 0xFF)
            call()
        torch.cuda.synchronize()
        capi.fno_profile_enable(False)
        stats = capi.fno_profile_read()
    finally:
        capi.fno_set_tensor_cores(prev)
    capi.fno_device_error(clear=True)
    return {t: v["total_ms"] * 1e3 / steps for t, v in stats.items()}


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--out", default=None)
    ap.add_argument("--workloads", nargs="*", default=None)
    args = ap.parse_args()
    capi.load()
    lines = ["| workload (block shape) | kernel path | kernel | us per call |", "|---|---|---|---|"]
    for name in args.workloads or synth.WORKLOAD_ORDER:
        wl = synth.WORKLOADS[name]
        for path, label in PATHS.items():
            per = _time_block(wl, path, args.steps)
            total = 0.0
            for tag, us in sorted(per.items(), key=lambda kv: -kv[1]):
                lines.append(f"| {name} | {path}: {label} | {tag} | {us:.1f} |")
                total += us
            lines.append(f"| {name} | {path}: {label} | **block fwd + bwd** | **{total:.1f}** |")
    text = "\n".join(lines)
    print(text)
    if args.out:
        with open(args.out, "w") as f:
            f.write(text + "\n")


if __name__ == "__main__":
    main()
