"""Training loop with a precision schedule, over the library's C ABI.

Mixed-precision training of neural operators ("Guaranteed approximation
bounds and efficient mixed-precision training for neural operators",
summary) ends with a precision schedule: training runs in half precision
(fp16 or bf16 storage with float32 accumulation, tanh pre-activation for
fp16) and moves to full precision part-way through.  The page fixes neither
the optimiser nor the switch point; here they are Adam with decoupled weight
decay on float32 master weights, and a list of (first step, storage dtype)
phases, by default half precision for the first half of the steps.

All weights live in flat device buffers with one 16-byte aligned slot per
parameter: the float32 master copy, the Adam moments, the float32 gradient
that ``fno_backward`` writes, and the copy in the current storage dtype that
the forward reads.  A step is forward, MSE and backward in that step's
dtype, the all-reduce of the gradient (data parallelism over the batch: one
collective per gradient group, started as soon as the backward has finished
the group, so that it overlaps the backward of the earlier layers), then one
fused ``fno_adam_step`` launch that updates the master copy
and writes the next step's weights in the next step's dtype.

Host logic only: every arithmetic step runs in ``libfno.so``; torch provides
the buffers, the stream and ``torch.distributed``.
"""

from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from . import capi

STORAGE_DTYPES = ("f32", "f16", "bf16")
ALIGN = 8   # elements per slot boundary: 16 bytes in every storage dtype


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


class PrecisionSchedule:
    """Storage dtype per training step: phases ``[(first step, dtype), ...]``."""

    def __init__(self, phases: Sequence[Tuple[int, str]]):
        phases = [(int(s), str(d)) for s, d in phases]
        if not phases or phases[0][0] != 0:
            raise ValueError("the first phase must start at step 0")
        starts = [s for s, _ in phases]
        if any(b <= a for a, b in zip(starts, starts[1:])):
            raise ValueError("phase starts must increase")
        for _, d in phases:
            if d not in STORAGE_DTYPES:
                raise ValueError(f"unknown storage dtype {d!r}")
        self.phases: List[Tuple[int, str]] = phases

    @classmethod
    def mixed_then_full(cls, total_steps: int, half: str = "bf16",
                        switch_fraction: float = 0.5) -> "PrecisionSchedule":
        """Half precision for the first ``switch_fraction`` of the steps, then f32."""
        if half not in ("f16", "bf16"):
            raise ValueError("half must be 'f16' or 'bf16'")
        switch = int(round(total_steps * switch_fraction))
        if switch <= 0:
            return cls([(0, "f32")])
        if switch >= total_steps:
            return cls([(0, half)])
        return cls([(0, half), (switch, "f32")])

    def dtype_at(self, step: int) -> str:
        if step < 0:
            raise ValueError("step < 0")
        current = self.phases[0][1]
        for start, dtype in self.phases:
            if start <= step:
                current = dtype
        return current


class ParamLayout:
    """Slots of the network's parameters in one flat buffer.

    Order: P, p, then per layer R[l], W[l], b[l], then Q1, q1, Q2, q2, with
    the shapes of ``fno_params`` (R as [width][width][|K|][2] (re, im)).  Every
    slot starts at a multiple of ``ALIGN`` elements; the gaps stay zero.  The
    parameters of each gradient group the backward finishes together (the
    projection, each layer, the lift) are one contiguous range, so each group's
    all-reduce is one collective on a view of the flat gradient.
    """

    def __init__(self, in_channels: int, width: int, hidden: int, out_channels: int,
                 n_layers: int, n_modes: int):
        self.n_layers = n_layers
        entries = [("P", None, (width, in_channels)), ("p", None, (width,))]
        for l in range(n_layers):
            entries += [("R", l, (width, width, n_modes, 2)), ("W", l, (width, width)),
                        ("b", l, (width,))]
        entries += [("Q1", None, (hidden, width)), ("q1", None, (hidden,)),
                    ("Q2", None, (out_channels, hidden)), ("q2", None, (out_channels,))]
        self.slots = []
        off = 0
        for key, layer, shape in entries:
            size = int(np.prod(shape))
            self.slots.append((key, layer, shape, off, size))
            off += (size + ALIGN - 1) // ALIGN * ALIGN
        self.total = off

    def _start(self, key: str, layer=None) -> int:
        for k, l, _, off, _ in self.slots:
            if k == key and l == layer:
                return off
        raise KeyError(key)

    def buckets(self) -> List[Tuple[int, int]]:
        """[lo, hi) element ranges of the gradient groups in the order the
        backward finishes them (fno_backward_ready): the projection, the layers
        from the last to the first, the lift.  Together they tile [0, total)."""
        L = self.n_layers
        starts = [self._start("R", l) for l in range(L)] + [self._start("Q1")]
        out = [(starts[L], self.total)]
        for l in range(L - 1, -1, -1):
            out.append((starts[l], starts[l + 1]))
        out.append((0, starts[0]))
        return out

    def views(self, flat) -> Dict[str, object]:
        """Per-parameter views of ``flat`` (lists for R, W, b)."""
        out: Dict[str, object] = {"R": [], "W": [], "b": []}
        for key, layer, shape, off, size in self.slots:
            v = flat[off:off + size].view(*shape)
            if layer is None:
                out[key] = v
            else:
                out[key].append(v)
        return out

    def pack(self, params: Dict[str, object], flat) -> None:
        """Copy a parameter dict (NumPy or torch; complex R allowed) into ``flat``."""
        import torch
        for key, layer, shape, off, size in self.slots:
            val = params[key] if layer is None else params[key][layer]
            arr = np.asarray(val.detach().cpu().numpy() if isinstance(val, torch.Tensor) else val)
            if np.iscomplexobj(arr):
                arr = np.stack([arr.real, arr.imag], -1)
            if tuple(arr.shape) != tuple(shape):
                raise ValueError(f"{key}{'' if layer is None else [layer]}: shape {arr.shape}, "
                                 f"expected {shape}")
            flat[off:off + size].copy_(torch.from_numpy(np.ascontiguousarray(arr, np.float32))
                                       .reshape(-1))

    def unpack(self, flat) -> Dict[str, object]:
        """NumPy float64 parameter dict from ``flat`` (R complex)."""
        host = flat.detach().float().cpu().numpy().astype(np.float64)
        out: Dict[str, object] = {"R": [], "W": [], "b": []}
        for key, layer, shape, off, size in self.slots:
            arr = host[off:off + size].reshape(shape)
            if key == "R":
                arr = arr[..., 0] + 1j * arr[..., 1]
            if layer is None:
                out[key] = arr
            else:
                out[key].append(arr)
        return out


class Trainer:
    """Adam training of the FNO network under a precision schedule.

    ``params``: the network's parameters (``P, p, R, W, b, Q1, q1, Q2, q2``;
    NumPy or torch; R complex or [..][2]); they become the float32 master copy.
    ``process_group``: with more than one rank the flat gradient is summed by
    one all-reduce and the optimiser averages it (every rank holds an equal
    share of the global batch, so this is the gradient of the global-mean MSE).
    """

    def __init__(self, grid: Sequence[int], modes: Sequence[int], in_channels: int, width: int,
                 params: Dict[str, object], schedule: PrecisionSchedule, hidden: int = 128,
                 out_channels: int = 1, n_layers: int = 4, flags: int = 0, lr: float = 1e-3,
                 betas: Tuple[float, float] = (0.9, 0.999), eps: float = 1e-8,
                 weight_decay: float = 0.0, device=None, process_group=None):
        import torch
        self.grid, self.modes = tuple(int(n) for n in grid), tuple(int(m) for m in modes)
        self.in_channels, self.width, self.hidden = in_channels, width, hidden
        self.out_channels, self.n_layers, self.flags = out_channels, n_layers, flags
        self.schedule = schedule
        self.lr, self.betas, self.eps, self.weight_decay = lr, betas, eps, weight_decay
        self.device = torch.device(device) if device is not None else \
            torch.device("cuda", torch.cuda.current_device())
        self.pg = process_group
        self.layout = ParamLayout(in_channels, width, hidden, out_channels, n_layers,
                                  capi.num_modes(self.grid, self.modes))
        n = self.layout.total
        self.master = torch.zeros(n, dtype=torch.float32, device=self.device)
        self.layout.pack(params, self.master)
        self.m = torch.zeros_like(self.master)
        self.v = torch.zeros_like(self.master)
        self.grad = torch.zeros_like(self.master)
        self.step_count = 0
        self.dtype: Optional[str] = None
        self.weights = None
        self._bufs: Dict[Tuple[str, int], Dict[str, object]] = {}
        self._buckets = self.layout.buckets()
        self._ready = None        # per-group events and the collective stream (CUDA, world > 1)
        self._comm = None

    # ---------------------------------------------------------------- helpers
    def _desc(self, dtype: str, batch: int):
        return capi.net_desc(batch, self.grid, self.modes, self.in_channels, self.width,
                             self.hidden, self.out_channels, self.n_layers, dtype, self.flags)

    def _buffers(self, dtype: str, batch: int) -> Dict[str, object]:
        import torch
        key = (dtype, batch)
        if key not in self._bufs:
            d = self._desc(dtype, batch)
            u_shape = (batch, self.out_channels) + self.grid
            self._bufs[key] = {
                "saves": torch.empty(capi.fno_net_saves_size(d), dtype=torch.uint8,
                                     device=self.device),
                "ws_fwd": torch.empty(capi.fno_net_workspace_size(d, capi.FNO_OP_NET_FWD),
                                      dtype=torch.uint8, device=self.device),
                "ws_bwd": torch.empty(capi.fno_net_workspace_size(d, capi.FNO_OP_NET_BWD),
                                      dtype=torch.uint8, device=self.device),
                "u": torch.empty(u_shape, dtype=torch_dtype(dtype), device=self.device),
                "du": torch.empty(u_shape, dtype=torch_dtype(dtype), device=self.device),
                "loss": torch.zeros(1, dtype=torch.float32, device=self.device),
            }
        return self._bufs[key]

    def _weights_for(self, dtype: str):
        import torch
        if self.dtype != dtype:
            w = torch.empty(self.layout.total, dtype=torch_dtype(dtype), device=self.device)
            capi.fno_adam_step(self.master, None, None, None, w, 1, 0.0)   # copy only
            self.weights, self.dtype = w, dtype
        return self.weights

    def params(self) -> Dict[str, object]:
        """The float32 master weights as a NumPy float64 dict (R complex)."""
        return self.layout.unpack(self.master)

    def state_dict(self) -> Dict[str, object]:
        """Everything a resumed run needs: master weights, Adam moments, step
        count, schedule and hyper-parameters (tensors copied to the host)."""
        return {"master": self.master.detach().cpu().clone(), "m": self.m.detach().cpu().clone(),
                "v": self.v.detach().cpu().clone(), "step": self.step_count,
                "phases": list(self.schedule.phases), "lr": self.lr, "betas": tuple(self.betas),
                "eps": self.eps, "weight_decay": self.weight_decay, "slots": self.layout.total}

    def load_state_dict(self, state: Dict[str, object]) -> None:
        """Resume from :meth:`state_dict` (same network shape)."""
        if int(state["slots"]) != self.layout.total:
            raise ValueError("checkpoint is of a different network shape")
        self.master.copy_(state["master"])
        self.m.copy_(state["m"])
        self.v.copy_(state["v"])
        self.step_count = int(state["step"])
        self.schedule = PrecisionSchedule(state["phases"])
        self.lr, self.betas = float(state["lr"]), tuple(state["betas"])
        self.eps, self.weight_decay = float(state["eps"]), float(state["weight_decay"])
        self.dtype, self.weights = None, None     # the next step copies the master afresh

    def _allreduce_buckets(self) -> None:
        """Sum every gradient group over the process group, one collective per
        group in the order the backward finishes them (on CUDA: on the
        collective stream, each after its group's ready event)."""
        import torch
        import torch.distributed as dist
        if self._ready is None:
            for lo, hi in self._buckets:
                dist.all_reduce(self.grad[lo:hi], group=self.pg)
            return
        for (lo, hi), ev in zip(self._buckets, self._ready):
            self._comm.wait_event(ev)
            with torch.cuda.stream(self._comm):
                dist.all_reduce(self.grad[lo:hi], group=self.pg)
        torch.cuda.current_stream(self.device).wait_stream(self._comm)

    # ------------------------------------------------------------------- step
    def step(self, a, target):
        """One step on a batch: ``a`` [B][in][grid], ``target`` [B][out][grid]
        (device tensors, any float dtype; cast to the step's storage dtype).
        Returns this step's loss as a float32 device tensor of one element."""
        import torch
        dt = self.schedule.dtype_at(self.step_count)
        w = self._weights_for(dt)
        a_s = a.to(device=self.device, dtype=torch_dtype(dt)).contiguous()
        t_s = target.to(device=self.device, dtype=torch_dtype(dt)).contiguous()
        batch = int(a_s.shape[0])
        d = self._desc(dt, batch)
        b = self._buffers(dt, batch)
        cp = capi.make_params(self.layout.views(w))
        cg = capi.make_grads(self.layout.views(self.grad))
        capi.fno_forward(d, a_s, cp, b["u"], b["saves"], ws=b["ws_fwd"])
        capi.fno_mse(b["u"], t_s, b["loss"], b["du"], dtype=dt)
        scale = 1.0
        world = 1
        if self.pg is not None:
            import torch.distributed as dist
            world = dist.get_world_size(self.pg)
        if world > 1 and self.device.type == "cuda":
            # each gradient group's all-reduce starts on the collective stream as
            # soon as the backward has finished that group, overlapping the
            # backward of the earlier layers
            if self._ready is None:
                self._ready = [torch.cuda.Event() for _ in self._buckets]
                self._comm = torch.cuda.Stream(device=self.device)
            capi.fno_backward(d, a_s, cp, b["saves"], b["du"], cg, ws=b["ws_bwd"],
                              ready=self._ready)
            self._allreduce_buckets()
            scale = 1.0 / world
        else:
            capi.fno_backward(d, a_s, cp, b["saves"], b["du"], cg, ws=b["ws_bwd"])
            if world > 1:
                self._allreduce_buckets()
                scale = 1.0 / world
        self.step_count += 1
        nxt = self.schedule.dtype_at(self.step_count)
        out = w if nxt == dt else torch.empty(self.layout.total, dtype=torch_dtype(nxt),
                                              device=self.device)
        capi.fno_adam_step(self.master, self.m, self.v, self.grad, out, self.step_count, self.lr,
                           self.betas[0], self.betas[1], self.eps, self.weight_decay, scale)
        self.weights, self.dtype = out, nxt
        return b["loss"].clone()
