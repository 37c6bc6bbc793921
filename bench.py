#!/usr/bin/env python
"""Benchmark of the FNO hot path on B200: one step = one forward pass of the 2D
FNO network (lift 3->32, four spectral blocks of width 32 with 16x16 modes on a
256x256 grid, projection 32->128->1, float32) over a batch of 16 synthetic
log-resistivity fields, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fno|reference]

Prints one JSON line (rank 0).  With N > 1 (launched by torch.distributed.run)
every rank runs its own batch of 16 (weak scaling, batch-sharded data
parallelism: the forward has no exchange step, so there is no collective on
the data path); the step time is the maximum over ranks.

``--impl reference`` times the CPU float64 oracle instead (rank 0 only; one
sample of the batch per step).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FNO block samples/sec at 1 B200; achieved HBM GB/s & tensor-pipe util vs peak"
DEFAULT_WORKLOAD = "fno2d_f32_b16_w32_256sq_m16"
FLUSH_BYTES = 512 << 20          # > 126 MB L2: written between timed steps
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("fno", "reference"), default="fno")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bound on the CPU-oracle sample of the fno arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the forward step's kernels one by one instead of replaying "
                         "them as a captured CUDA graph")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--kernel-path", type=int, choices=(0, 1, 2, 3), default=1,
                    help="library kernel selection (fno_set_tensor_cores): 1 default, "
                         "3 tensor-core DFT-matrix pipelines, 2 tensor cores without "
                         "pipelines, 0 CUDA cores")
    return ap.parse_args()


def resolve_workload(args):
    import dataclasses

    from fourier_neural_spectral_fno_b200 import synth
    if args.workload not in synth.WORKLOADS:
        raise SystemExit(f"unknown workload {args.workload!r}; one of: "
                         + ", ".join(synth.WORKLOAD_ORDER))
    wl = synth.WORKLOADS[args.workload]
    if wl.kind != "network":
        nets = [n for n in synth.WORKLOAD_ORDER if synth.WORKLOADS[n].kind == "network"]
        raise SystemExit(f"workload {args.workload!r} is a single-block parity case; bench.py "
                         "times network workloads: " + ", ".join(nets))
    if args.batch is not None:
        if args.batch < 1:
            raise SystemExit("--batch must be >= 1")
        wl = dataclasses.replace(wl, batch=args.batch)
    return wl


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
            self.pg = dist

    def barrier(self):
        if self.pg:
            import torch
            if torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# --------------------------------------------------------------------------
# clocks (NVML, read only)
# --------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and throttle reasons every few ms while running."""

    def __init__(self, index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # pragma: no cover - no NVML
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [n for bit, n in _REASONS.items() if self.reasons & bit]}


# --------------------------------------------------------------------------
# the workload
# --------------------------------------------------------------------------

def workload_config(wl, n_gpus):
    return {"workload": wl.name, "description": wl.description, "batch_per_gpu": wl.batch,
            "global_batch": wl.batch * n_gpus, "grid": list(wl.grid), "modes": list(wl.modes),
            "width": wl.width, "in_channels": wl.in_ch, "hidden": wl.hidden,
            "blocks": wl.n_layers, "storage": wl.dtype,
            "l2": "flushed between timed steps (512 MiB write outside the step events)",
            "step": ("training: forward + MSE + backward" +
                     (" + per-group NCCL gradient all-reduce overlapping the backward"
                      if n_gpus > 1 else "") + " + Adam step"
                     if wl.backward and wl.kind == "network" else "forward"),
            "parallelism": (f"dp{n_gpus} (batch-sharded" +
                            (", gradient all-reduce)" if wl.backward and wl.kind == "network"
                             and n_gpus > 1 else ", no data-path collective)"))}


def algorithmic_bytes(tag: str, wl) -> float:
    """Bytes a kernel must move per launch (each operand once) for the workload."""
    s = 4 if wl.dtype == "f32" else 2
    act = wl.batch * wl.width * wl.points * s
    k = wl.modes[-1]
    for m in wl.modes[:-1]:
        k *= 2 * m
    spec = wl.batch * wl.width * k * 8
    r = wl.width * wl.width * k * 2 * s
    rows = wl.batch * wl.points // wl.grid[-1]       # (sample, grid row) pairs
    img = rows * (2 if wl.dtype == "f32" else 1) * wl.width * 2 * wl.modes[-1] * s
    table = {
        "fwd_transform": act + spec,                 # read x, write spectrum
        "fwd_fft": act + spec,
        "fwd_plane": act + spec,
        "fwd_plane_dz": 2 * act + spec,
        "inv_slab_img": spec + img,                  # read yhat, write the B images
        "epi_block_fwd": 2 * act + spec,             # read x, write y, read spectrum
        "mix_fwd": 2 * spec + r,
        "lift": wl.batch * wl.in_ch * wl.points * s + act,
        "proj_fwd": act + wl.batch * wl.out_ch * wl.points * s,
    }
    for base in ("fwd_transform", "epi_block_fwd", "proj_fwd"):
        table[base + "_tc"] = table[base]
    table["epi_block_fwd_pipe"] = table["epi_block_fwd"]
    table["epi_block_bwd"] = 4 * act + spec         # read dy, pre, x; write dx; read spectrum
    table["fwd_transform_dz"] = 2 * act + spec      # read dy, pre; write spectrum
    table["fwd_transform_tc_dz"] = table["fwd_transform_dz"]
    table["proj_bwd"] = 2 * act + 2 * wl.batch * wl.out_ch * wl.points * s
    table["fwd_transform_pipe"] = table["fwd_transform"]
    table["proj_fwd_pipe"] = table["proj_fwd"]
    # tensor-core backward: read dy, pre, x and the slab-inverted dxhat rows
    # ([B][C][rows][m_L] complex), write dx
    table["epi_block_bwd_pipe"] = 4 * act + rows * wl.width * wl.modes[-1] * 8
    table["proj_bwd_pipe"] = table["proj_bwd"]
    table["mix_fwd_tc"] = table["mix_fwd"]          # read spectrum and R, write spectrum
    table["mix_bwd_dx"] = table["mix_bwd_dx_tc"] = table["mix_fwd"]
    table["mix_bwd_dr"] = table["mix_bwd_dr_tc"] = 2 * spec + 2 * wl.width * wl.width * k * 4
    return float(table.get(tag, 0.0))


def kernel_source_sha(tag: str) -> str:
    files = {"fwd_transform": "transform.cu", "fwd_finish": "transform.cu",
             "epi_block_fwd": "epilogue.cu", "mix_fwd": "mix.cu", "lift": "net.cu",
             "proj_fwd": "net.cu", "fwd_transform_tc": "transform_tc.cu",
             "epi_block_fwd_tc": "epilogue_tc.cu", "inv_slab": "epilogue_tc.cu",
             "proj_fwd_tc": "net_tc.cu", "epi_block_fwd_pipe": "epilogue_pipe.cu",
             "fwd_transform_pipe": "transform_pipe.cu", "proj_fwd_pipe": "proj_pipe.cu",
             "epi_block_bwd": "epilogue.cu", "proj_bwd": "net.cu",
             "fwd_transform_tc_dz": "transform_tc.cu", "fwd_transform_dz": "transform.cu",
             "fwd_fft": "transform_fft.cu", "fwd_fft_dz": "transform_fft.cu",
             "fwd_plane": "transform_plane.cu", "fwd_plane_dz": "transform_plane.cu",
             "inv_slab_img": "spec_mid.cu", "inv_slab_fft": "spec_mid.cu",
             "epi_block_bwd_pipe": "epilogue_pipe.cu", "proj_bwd_pipe": "proj_pipe.cu",
             "mix_fwd_tc": "mix_tc.cu", "mix_bwd_dx_tc": "mix_tc.cu", "lift_bwd": "net.cu",
             "mix_bwd_dx": "mix.cu", "mix_bwd_dr": "mix.cu", "mix_bwd_dr_tc": "mix_tc.cu",
             "epi_spec": "epilogue.cu",
             "epi_spec_bwd": "epilogue.cu"}
    path = os.path.join(ROOT, "fourier_neural_spectral_fno_b200", "csrc", files.get(tag, ""))
    if not os.path.isfile(path):
        return ""
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def measured_traffic(tag: str, wl):
    """ncu DRAM bytes per launch from profiles/traffic.json, or None when absent
    or when the kernel's source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[wl.name][tag]
    except Exception:
        return None
    if rec.get("source_sha") != kernel_source_sha(tag):
        return None
    return rec.get("bytes_per_launch")


FP32_LANES_PER_SM = 128      # FP32 FMA lanes per SM: 4 sub-partitions x 32
FALLBACK_SM_MHZ = 1965.0


def alu_peak_tflops(n_sms: int):
    """FP32 CUDA-core peak: 2 FLOP per FMA x FMA lanes x SMs x maximum SM clock
    (the clock from MEASURED_PEAKS.json, else the B200's 1965 MHz)."""
    try:
        mhz = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["sm_max_mhz"])
        src = "derived: measured max SM clock"
    except Exception:
        mhz, src = FALLBACK_SM_MHZ, "derived: nominal max SM clock"
    return 2.0 * FP32_LANES_PER_SM * n_sms * mhz * 1e6 / 1e12, src


def algorithmic_flops(tag: str, wl) -> float:
    """FP32 FLOPs per launch of the CUDA-core kernels whose bound is arithmetic
    (0 for the others): each contraction's multiply-adds, two FLOPs apiece."""
    pts = wl.batch * wl.points
    c, m_l, h = wl.width, wl.modes[-1], wl.hidden
    table = {
        # last-axis inverse of dxhat (a complex multiply-add per mode and channel: 4 FLOPs),
        # dx = W^T dz and dW = dz x^T (2 FLOPs per channel pair each)
        "epi_block_bwd": pts * (4 * m_l * c + 4 * c * c),
        # hidden layer recomputed (Q1 v), dv = Q1^T dh, dQ1 = dh v^T, dQ2 = du g^T
        "proj_bwd": pts * (6 * h * c + 2 * h * wl.out_ch),
    }
    return float(table.get(tag, 0.0))


def roofline_record(dom: str, avg_ms: float, wl, n_sms: int) -> dict:
    """The roofline object of the dominant kernel: against the FP32 CUDA-core
    peak for the arithmetic-bound CUDA-core kernels, else against the measured
    HBM copy bandwidth."""
    alg = algorithmic_bytes(dom, wl)
    hbm, hbm_src = hbm_peak()
    gbs = alg / (avg_ms / 1e3) / 1e9 if alg else None
    flops = algorithmic_flops(dom, wl)
    if flops:
        peak, src = alu_peak_tflops(n_sms)
        achieved = flops / (avg_ms / 1e3) / 1e12
        return {"kernel": dom, "bound": "alu", "achieved": achieved, "peak": peak,
                "peak_source": f"{src} x {FP32_LANES_PER_SM} FP32 lanes x {n_sms} SMs x 2",
                "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": measured_traffic(dom, wl), "avg_launch_ms": avg_ms,
                "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": alg,
                "hbm_view": {"achieved": gbs, "peak": hbm, "unit": "GB/s",
                             "frac": (gbs / hbm) if gbs else None}}
    return {"kernel": dom, "bound": "hbm", "achieved": gbs, "peak": hbm,
            "peak_source": hbm_src,
            "unit": "GB/s", "frac": (gbs / hbm) if gbs else None,
            "traffic": measured_traffic(dom, wl), "avg_launch_ms": avg_ms,
            "algorithmic_bytes_per_launch": alg}


NON_BLOCK_TAGS = ("lift", "proj_fwd", "proj_fwd_tc", "proj_fwd_pipe")


def block_roofline_record(stats: dict, steps: int, wl) -> dict:
    """The spectral block as a whole (forward workloads): its algorithmic HBM
    bytes (x read once, y written once, R read once) over the summed device time
    of every kernel that belongs to the blocks, per block, against the measured
    copy bandwidth; ncu DRAM bytes per block where every block kernel has a
    current capture."""
    s = 4 if wl.dtype == "f32" else 2
    k = wl.modes[-1]
    for m in wl.modes[:-1]:
        k *= 2 * m
    alg = 2 * wl.batch * wl.width * wl.points * s + wl.width * wl.width * k * 2 * s
    tags = [t for t in stats if t not in NON_BLOCK_TAGS]
    ms = sum(stats[t]["total_ms"] for t in tags) / steps / wl.n_layers
    hbm, src = hbm_peak()
    gbs = alg / (ms / 1e3) / 1e9
    traffic = 0.0
    for t in tags:
        per_launch = measured_traffic(t, wl)
        if per_launch is None:
            traffic = None
            break
        traffic += per_launch * stats[t]["launches"] / steps / wl.n_layers
    return {"scope": "one spectral block (all its kernels)", "bound": "hbm", "achieved": gbs,
            "peak": hbm, "peak_source": src,
            "unit": "GB/s", "frac": gbs / hbm, "block_ms": ms,
            "algorithmic_bytes_per_block": float(alg), "traffic": traffic,
            "kernels": sorted(tags)}


def hbm_peak():
    """The copy bandwidth the HBM fractions divide by, and where it came from."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return (float(json.load(open(path))["hbm_gbs"]),
                "measured (MEASURED_PEAKS.json hbm_gbs, a STREAM-style copy)")
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (MEASURED_PEAKS.json absent; an earlier copy measurement)"


def cpu_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(i.get("num_threads", 1) for i in info) if info else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_samples(wl, inp, n_samples):
    """The oracle's step on the first n_samples of the batch: the forward, and
    for training workloads the MSE and the backward as well."""
    import oracle as O
    a = inp["a"][:n_samples]
    if not (wl.backward and wl.kind == "network"):
        return O.forward(a, inp["params"], wl.modes)
    u, sv = O.forward(a, inp["params"], wl.modes, save=True)
    _, du = O.mse(u, inp["target"][:n_samples])
    return O.backward(a, inp["params"], sv, du, wl.modes)


def _one_sample(inp, i):
    one = {"a": inp["a"][i:i + 1], "params": inp["params"]}
    if inp.get("target") is not None:
        one["target"] = inp["target"][i:i + 1]
    return one


def cpu_baseline(wl, inp, seconds):
    """The oracle on a bounded sample of the workload (whole samples, one at a
    time, until `seconds` of CPU work or the batch is done)."""
    done, t0 = 0, time.perf_counter()
    while done < wl.batch and (time.perf_counter() - t0) < seconds:
        oracle_samples(wl, _one_sample(inp, done), 1)
        done += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "samples/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{done} of {wl.batch} samples of the workload, full grid, all blocks, "
                      f"float64 NumPy, {dt:.1f} s"}


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------

def run_reference(args, dist):
    from fourier_neural_spectral_fno_b200 import synth
    wl = resolve_workload(args)
    if dist.rank != 0:
        return
    inp = synth.make_network_inputs(wl)
    for i in range(args.warmup):
        oracle_samples(wl, _one_sample(inp, i % wl.batch), 1)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_samples(wl, _one_sample(inp, i % wl.batch), 1)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    cores = cpu_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "samples/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": "samples/s", "cores": cores, "kind": "oracle",
                             "sample": "one sample of the batch per step (full grid, all blocks)"},
            "e2e": {"value": value, "unit": "samples/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_fno(args, dist):
    import numpy as np
    import torch

    from fourier_neural_spectral_fno_b200 import capi, synth

    wl = resolve_workload(args)
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    capi.load()
    capi.fno_set_tensor_cores(args.kernel_path)

    inp = synth.make_network_inputs(wl)
    tdt = torch.float32 if wl.dtype == "f32" else (torch.float16 if wl.dtype == "f16" else torch.bfloat16)

    def up(v):
        v = np.asarray(v)
        if np.iscomplexobj(v):
            v = np.stack([v.real, v.imag], -1)
        return torch.from_numpy(np.ascontiguousarray(v)).to(dev).to(tdt)

    params = {k: ([up(x) for x in v] if isinstance(v, list) else up(v))
              for k, v in inp["params"].items()}
    cp = capi.make_params(params)
    desc = capi.net_desc(wl.batch, wl.grid, wl.modes, wl.in_ch, wl.width, wl.hidden, wl.out_ch,
                         wl.n_layers, wl.dtype, capi.FNO_TANH_PREACT if wl.tanh else 0)
    a = up(inp["a"])
    u = torch.empty((wl.batch, wl.out_ch) + wl.grid, dtype=tdt, device=dev)
    train = wl.backward and wl.kind == "network"
    ws = None if train else torch.empty(capi.fno_net_workspace_size(desc, capi.FNO_OP_NET_FWD),
                                        dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    if train:
        # one training step of the library's Trainer: forward (keeping the
        # saves), MSE against the target, backward into the flat float32
        # gradient, with several ranks the per-group NCCL all-reduces that
        # overlap the backward, and the fused Adam step that writes the next
        # step's weights
        import torch.distributed as tdist

        from fourier_neural_spectral_fno_b200 import train as fno_train
        target = up(inp["target"])
        trainer = fno_train.Trainer(
            wl.grid, wl.modes, wl.in_ch, wl.width, inp["params"],
            fno_train.PrecisionSchedule([(0, wl.dtype)]), hidden=wl.hidden,
            out_channels=wl.out_ch, n_layers=wl.n_layers,
            flags=capi.FNO_TANH_PREACT if wl.tanh else 0, lr=1e-4, device=dev,
            process_group=tdist.group.WORLD if dist.world > 1 else None)
        loss = torch.empty(1, dtype=torch.float32, device=dev)

        def step(a_in=a, t_in=target, u_out=None, loss_out=loss):
            loss_out.copy_(trainer.step(a_in, t_in))
    else:
        target = loss = None

        def step(a_in=a, t_in=None, u_out=u, loss_out=None):
            capi.fno_forward(desc, a_in, cp, u_out, None, ws, torch.cuda.current_stream())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # the forward step as a CUDA graph: its ~18 dependent launches are replayed
    # without a host launch between kernels (one graph per set of buffers)
    use_graph = not train and not args.no_graph
    graphs = {}

    def graph_step(a_in, u_out):
        key = (a_in.data_ptr(), u_out.data_ptr())
        if key not in graphs:
            gr = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            with torch.cuda.graph(gr, capture_error_mode="relaxed"):
                step(a_in, None, u_out, None)
            torch.cuda.synchronize()
            graphs[key] = gr
        graphs[key].replay()

    timed_step = (lambda: graph_step(a, u)) if use_graph else step
    if use_graph:
        for _ in range(args.warmup):
            timed_step()
        torch.cuda.synchronize()

    # ---- timed region: K steps, events around each step, L2 flushed between
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    reg0, reg1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        reg0.record()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record()
            timed_step()
            ends[i].record()
        reg1.record()
        torch.cuda.synchronize()
    dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = dist.max(sum(step_ms) / len(step_ms))
    region_ms = dist.max(reg0.elapsed_time(reg1))
    value = dist.world * wl.batch / (ms / 1e3)

    # ---- per-kernel device time (second pass, profiling events on)
    capi.fno_profile_enable(True)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    capi.fno_profile_enable(False)
    stats = capi.fno_profile_read()
    launches = sum(v["launches"] for v in stats.values()) // args.steps   # the library's kernels
    dom = max(stats, key=lambda t: stats[t]["total_ms"])
    avg_ms = stats[dom]["total_ms"] / stats[dom]["launches"]
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    roofline = roofline_record(dom, avg_ms, wl, n_sms)
    if not train:
        roofline["block"] = block_roofline_record(stats, args.steps, wl)
    per_step = {t: round(v["total_ms"] / args.steps, 4) for t, v in sorted(
        stats.items(), key=lambda kv: -kv[1]["total_ms"])}

    # ---- end to end through the public API with host buffers.  Every step
    # copies its inputs from pinned host memory and the host reads its result;
    # two buffer slots let step i+1's input copy and step i's result copy run on
    # a copy stream while the compute stream works (the stream order still
    # makes each step wait for its own inputs).
    ins = [a, target] if train else [a]            # the step's inputs
    out = loss if train else u                     # the step's result the host reads
    ins_host = []
    for t in ins:
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t.cpu())
        ins_host.append(h)
    slots = []
    for _ in range(2):
        sl = {"ins": [torch.empty_like(t) for t in ins], "out": torch.empty_like(out),
              "host": torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
              "in_ev": torch.cuda.Event(), "done_ev": torch.cuda.Event(),
              "out_ev": torch.cuda.Event()}
        slots.append(sl)
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)

    def e2e_step(i):
        # inputs in on one copy stream, results out on another, so that step
        # i + 1's input copy never queues behind step i's result copy (which
        # waits for step i's compute)
        sl = slots[i & 1]
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(sl["out_ev"])     # slot free: step i-2 fully done
            for t, h in zip(sl["ins"], ins_host):
                t.copy_(h, non_blocking=True)
            sl["in_ev"].record(h2d_stream)
        stream.wait_event(sl["in_ev"])
        if train:
            step(sl["ins"][0], sl["ins"][1], None, sl["out"])
        elif use_graph:
            graph_step(sl["ins"][0], sl["out"])
        else:
            step(sl["ins"][0], None, sl["out"], None)
        sl["done_ev"].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(sl["done_ev"])
            sl["host"].copy_(sl["out"], non_blocking=True)
            sl["out_ev"].record(d2h_stream)

    def host_read(i):
        sl = slots[i & 1]
        sl["out_ev"].synchronize()
        return float(sl["host"].view(-1)[0])        # the host reads the step's result

    e_steps = max(3, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
        host_read(i)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d_stream)
    for i in range(e_steps):
        e2e_step(i)
        if i >= 1:
            host_read(i - 1)
    host_read(e_steps - 1)
    e1.record(d2h_stream)
    torch.cuda.synchronize()
    e_ms = dist.max(e0.elapsed_time(e1) / e_steps)
    e2e = {"value": dist.world * wl.batch / (e_ms / 1e3), "unit": "samples/s",
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in ins),
           "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": e_ms,
           "copies": "pinned host buffers; H2D and D2H on two copy streams overlapping the "
                     "neighbouring steps' compute (two buffer slots)"}

    clocks = clk.summary()
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, inp, args.cpu_seconds)

    if dist.rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "samples/s", "n_gpus": dist.world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "region_ms_per_step_incl_flush": region_ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": wl.dtype, "data": "synthetic",
                "config": dict(workload_config(wl, dist.world), kernel_path=args.kernel_path,
                               cuda_graph=use_graph),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches * args.steps, "launches_per_step": launches,
                "clocks": clocks, "kernels_ms_per_step": per_step}
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)      # rank 0 only; no process group needed
        return
    dist.init("nccl")
    try:
        run_fno(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
