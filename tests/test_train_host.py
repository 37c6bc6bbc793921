"""Host logic of the training loop (CPU): the precision schedule and the flat
parameter layout."""

import numpy as np
import pytest
import torch

import oracle as O
from fourier_neural_spectral_fno_b200 import synth
from fourier_neural_spectral_fno_b200.train import ALIGN, ParamLayout, PrecisionSchedule


def test_schedule_phases_and_errors():
    s = PrecisionSchedule([(0, "bf16"), (3, "f32")])
    assert [s.dtype_at(t) for t in range(5)] == ["bf16"] * 3 + ["f32"] * 2
    for bad in ([], [(1, "f32")], [(0, "f32"), (0, "bf16")], [(0, "f64")]):
        with pytest.raises(ValueError):
            PrecisionSchedule(bad)


@pytest.mark.parametrize("total,frac,expect", [
    (10, 0.5, [(0, "bf16"), (5, "f32")]), (10, 0.0, [(0, "f32")]), (10, 1.0, [(0, "bf16")]),
    (7, 0.3, [(0, "bf16"), (2, "f32")]),
])
def test_mixed_then_full(total, frac, expect):
    assert PrecisionSchedule.mixed_then_full(total, "bf16", frac).phases == expect


@pytest.mark.parametrize("phases", [[(0, "f16")], [(0, "bf16"), (2, "f32")],
                                    [(0, "f32"), (1, "bf16"), (4, "f32")]])
def test_schedule_agrees_with_oracle_reading(phases):
    s = PrecisionSchedule(phases)
    assert [s.dtype_at(t) for t in range(8)] == [O.dtype_at(phases, t) for t in range(8)]


def test_layout_slots_are_aligned_and_disjoint():
    lay = ParamLayout(3, 6, 9, 2, 3, 40)
    prev_end = 0
    for key, layer, shape, off, size in lay.slots:
        assert off % ALIGN == 0 and off >= prev_end
        assert size == int(np.prod(shape))
        prev_end = off + size
    assert lay.total >= prev_end and lay.total % ALIGN == 0
    assert [k for k, *_ in lay.slots] == ["P", "p"] + ["R", "W", "b"] * 3 + \
        ["Q1", "q1", "Q2", "q2"]
    assert [l for _, l, *_ in lay.slots] == [None, None, 0, 0, 0, 1, 1, 1, 2, 2, 2] + [None] * 4


def test_layout_buckets_follow_the_backward_and_tile_the_buffer():
    lay = ParamLayout(3, 6, 9, 2, 3, 40)
    bk = lay.buckets()
    assert len(bk) == 3 + 2
    assert sorted(bk) == sorted(set(bk))
    # contiguous tiling of [0, total)
    edges = sorted(bk)
    assert edges[0][0] == 0 and edges[-1][1] == lay.total
    assert all(a[1] == b[0] for a, b in zip(edges, edges[1:]))
    # projection first, then layers 2, 1, 0, then the lift
    start = {(k, l): off for k, l, _, off, _ in lay.slots}
    assert bk[0] == (start[("Q1", None)], lay.total)
    assert bk[1][0] == start[("R", 2)] and bk[3][0] == start[("R", 0)]
    assert bk[-1] == (0, start[("R", 0)])
    # each bucket holds exactly its group's slots
    for (lo, hi), keys in zip(bk, [{"Q1", "q1", "Q2", "q2"}, {2}, {1}, {0}, {"P", "p"}]):
        inside = {(k, l) for k, l, _, off, size in lay.slots if lo <= off and off + size <= hi}
        if isinstance(next(iter(keys)), int):
            assert inside == {(k, next(iter(keys))) for k in ("R", "W", "b")}
        else:
            assert inside == {(k, None) for k in keys}


def test_layout_pack_unpack_round_trip():
    wl = synth.Workload("tiny", "network", "f32", 2, (16, 12), (4, 5), 6, in_ch=3, hidden=9,
                        n_layers=2, backward=True)
    params = synth.make_network_inputs(wl)["params"]
    lay = ParamLayout(3, 6, 9, 1, 2, synth._num_kept((16, 12), (4, 5)))
    flat = torch.zeros(lay.total)
    lay.pack(params, flat)
    back = lay.unpack(flat)
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        np.testing.assert_array_equal(back[key], np.float32(params[key]))
    for key in ("R", "W", "b"):
        for l in range(2):
            np.testing.assert_array_equal(back[key][l], np.asarray(params[key][l]).astype(
                np.complex64 if key == "R" else np.float32))
    views = lay.views(flat)
    n_modes = next(shape for k, l, shape, *_ in lay.slots if (k, l) == ("R", 1))[2]
    assert tuple(views["R"][1].shape) == (6, 6, n_modes, 2)
    # gaps between slots stay zero
    used = np.zeros(lay.total, bool)
    for *_, off, size in lay.slots:
        used[off:off + size] = True
    assert not flat.numpy()[~used].any()
    with pytest.raises(ValueError):
        lay.pack({**params, "P": np.zeros((2, 2))}, flat)


class _FakeLibrary:
    """Stand-in for the C ABI on the CPU: the same calls computed by the oracle,
    on CPU tensors, so that the trainer's host logic (slots, dtype switches,
    step numbers, buffers) runs without a GPU."""

    def __init__(self, modes):
        self.modes = modes
        self.saved = {}
        self.FNO_OP_NET_FWD, self.FNO_OP_NET_BWD = 4, 5
        self.calls = []

    @staticmethod
    def num_modes(grid, modes):
        return O.num_modes(grid, modes)

    @staticmethod
    def net_desc(batch, grid, modes, in_channels, width, hidden, out_channels, n_layers, dtype,
                 flags):
        return {"batch": batch, "dtype": dtype, "flags": flags}

    def fno_net_saves_size(self, d):
        return 64

    def fno_net_workspace_size(self, d, op):
        return 64

    @staticmethod
    def make_params(views):
        return views

    make_grads = make_params

    @staticmethod
    def _np(views):
        out = {}
        for key, val in views.items():
            conv = (lambda t: (t.float().numpy()[..., 0] + 1j * t.float().numpy()[..., 1])
                    if key == "R" else t.float().numpy().astype(np.float64))
            out[key] = [conv(t) for t in val] if isinstance(val, list) else conv(val)
        return out

    def fno_forward(self, d, a, params, u, saves, ws=None):
        self.calls.append(("forward", d["dtype"], str(a.dtype)))
        p = self._np(params)
        uu, sv = O.forward(a.float().numpy().astype(np.float64), p, self.modes, save=True)
        self.saved[saves.data_ptr()] = sv
        u.copy_(torch.from_numpy(uu))

    def fno_mse(self, u, t, loss, du, dtype="f32"):
        val, d = O.mse(u.float().numpy(), t.float().numpy())
        loss.fill_(val)
        du.copy_(torch.from_numpy(d))

    def fno_backward(self, d, a, params, saves, du, grads, ws=None):
        g = O.backward(a.float().numpy().astype(np.float64), self._np(params),
                       self.saved[saves.data_ptr()], du.float().numpy().astype(np.float64),
                       self.modes)
        for key, val in grads.items():
            for l, t in enumerate(val if isinstance(val, list) else [val]):
                src = g[key][l] if isinstance(val, list) else g[key]
                if key == "R":
                    src = np.stack([src.real, src.imag], -1)
                t.copy_(torch.from_numpy(np.asarray(src, np.float32)))

    def fno_adam_step(self, theta, m, v, grad, out, step, lr, beta1=0.9, beta2=0.999, eps=1e-8,
                      weight_decay=0.0, grad_scale=1.0):
        self.calls.append(("adam", None if grad is None else int(step), str(out.dtype)))
        if grad is not None:
            th, mm, vv = O.adam_update(theta.numpy(), m.numpy(), v.numpy(),
                                       grad.numpy().astype(np.float64) * grad_scale, step, lr,
                                       beta1, beta2, eps, weight_decay)
            theta.copy_(torch.from_numpy(th.astype(np.float32)))
            m.copy_(torch.from_numpy(mm.astype(np.float32)))
            v.copy_(torch.from_numpy(vv.astype(np.float32)))
        out.copy_(theta.to(out.dtype))


def test_trainer_host_logic_with_fake_library(monkeypatch):
    from fourier_neural_spectral_fno_b200 import train as T
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "bf16", 2, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    fake = _FakeLibrary(modes)
    monkeypatch.setattr(T, "capi", fake)
    phases, steps, lr = [(0, "bf16"), (2, "f32")], 4, 1e-2
    tr = T.Trainer(grid, modes, 3, 4, inp["params"], T.PrecisionSchedule(phases), hidden=5,
                   n_layers=2, lr=lr, device="cpu")
    a = torch.from_numpy(np.asarray(inp["a"], np.float32))
    t = torch.from_numpy(np.asarray(inp["target"], np.float32))
    losses = [float(tr.step(a, t)) for _ in range(steps)]
    ref, ref_losses = O.train(inp["a"], inp["target"], inp["params"], modes, phases, steps, lr)
    # the fake, like the library, stores u and du in the step's dtype (bf16 first),
    # which the float64 loop does not: losses and weights agree loosely here
    np.testing.assert_allclose(losses, ref_losses, rtol=1e-3)
    got = tr.params()
    for key in ("P", "Q1", "q2"):
        assert np.linalg.norm(got[key] - ref[key]) <= 1e-2 * np.linalg.norm(ref[key]), key
    assert np.linalg.norm(got["R"][1] - ref["R"][1]) <= 1e-2 * np.linalg.norm(ref["R"][1])
    # the initial copy, then one Adam per step with 1-based step numbers; the
    # copy written at step 2 is already float32 for the switched phase
    assert fake.calls[0] == ("adam", None, "torch.bfloat16")
    adams = [c for c in fake.calls[1:] if c[0] == "adam"]
    assert [c[1] for c in adams] == [1, 2, 3, 4]
    assert [c[2] for c in adams] == ["torch.bfloat16", "torch.float32", "torch.float32",
                                     "torch.float32"]
    fwd = [c for c in fake.calls if c[0] == "forward"]
    assert [c[1] for c in fwd] == ["bf16", "bf16", "f32", "f32"]
    assert [c[2] for c in fwd] == ["torch.bfloat16"] * 2 + ["torch.float32"] * 2


def test_trainer_f32_with_fake_library_matches_oracle_loop(monkeypatch):
    from fourier_neural_spectral_fno_b200 import train as T
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "f32", 2, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    monkeypatch.setattr(T, "capi", _FakeLibrary(modes))
    tr = T.Trainer(grid, modes, 3, 4, inp["params"], T.PrecisionSchedule([(0, "f32")]), hidden=5,
                   n_layers=2, lr=1e-2, weight_decay=0.1, device="cpu")
    a = torch.from_numpy(np.asarray(inp["a"], np.float32))
    t = torch.from_numpy(np.asarray(inp["target"], np.float32))
    losses = [float(tr.step(a, t)) for _ in range(3)]
    ref, ref_losses = O.train(inp["a"], inp["target"], inp["params"], modes, [(0, "f32")], 3, 1e-2,
                              weight_decay=0.1)
    np.testing.assert_allclose(losses, ref_losses, rtol=1e-6)
    got = tr.params()
    for key in ("P", "p", "Q1", "q1", "Q2", "q2"):
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-5, atol=1e-6, err_msg=key)
    for key in ("R", "W", "b"):
        for l in range(2):
            np.testing.assert_allclose(got[key][l], ref[key][l], rtol=1e-5, atol=1e-6)


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _dp_trainer_worker(rank, world, port, out_dir):
    import os

    import torch.distributed as dist

    from fourier_neural_spectral_fno_b200 import train as T
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        grid, modes = (8, 6), (2, 2)
        wl = synth.Workload("tiny", "network", "f32", 4, grid, modes, 4, in_ch=3, hidden=5,
                            n_layers=2, backward=True)
        inp = synth.make_network_inputs(wl)
        T.capi = _FakeLibrary(modes)
        tr = T.Trainer(grid, modes, 3, 4, inp["params"], T.PrecisionSchedule([(0, "f32")]),
                       hidden=5, n_layers=2, lr=1e-2, eps=1.0, device="cpu",
                       process_group=dist.group.WORLD)
        lo, hi = rank * 2, rank * 2 + 2          # equal shards of the batch of 4
        a = torch.from_numpy(np.asarray(inp["a"][lo:hi], np.float32))
        t = torch.from_numpy(np.asarray(inp["target"][lo:hi], np.float32))
        for _ in range(2):
            tr.step(a, t)
        np.save(os.path.join(out_dir, f"master{rank}.npy"), tr.master.numpy())
    finally:
        dist.destroy_process_group()


def test_trainer_data_parallel_matches_full_batch(tmp_path, monkeypatch):
    """Two gloo ranks with half the batch each, gradient all-reduce and the
    1/world scale in the optimiser: the same weights as one rank on the whole
    batch (the gradient of the global-mean MSE).  eps = 1 makes the step
    close to linear in the gradient, so a wrong gradient scale shows (Adam
    with a small eps would hide it)."""
    import torch.multiprocessing as mp

    from fourier_neural_spectral_fno_b200 import train as T
    world = 2
    mp.start_processes(_dp_trainer_worker, args=(world, _free_port(), str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    m0, m1 = np.load(tmp_path / "master0.npy"), np.load(tmp_path / "master1.npy")
    np.testing.assert_array_equal(m0, m1)     # every rank holds the same weights
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "f32", 4, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    monkeypatch.setattr(T, "capi", _FakeLibrary(modes))
    tr = T.Trainer(grid, modes, 3, 4, inp["params"], T.PrecisionSchedule([(0, "f32")]), hidden=5,
                   n_layers=2, lr=1e-2, eps=1.0, device="cpu")
    a = torch.from_numpy(np.asarray(inp["a"], np.float32))
    t = torch.from_numpy(np.asarray(inp["target"], np.float32))
    start = tr.master.numpy().copy()
    for _ in range(2):
        tr.step(a, t)
    moved = np.abs(tr.master.numpy() - start).max()
    assert moved > 1e-4                            # the steps are not negligible
    np.testing.assert_allclose(m0, tr.master.numpy(), rtol=1e-5, atol=1e-3 * moved)


def test_trainer_resume_from_state_dict(monkeypatch):
    """Two steps, a checkpoint, a fresh trainer that loads it and two more steps
    end where four uninterrupted steps end (across the precision switch)."""
    from fourier_neural_spectral_fno_b200 import train as T
    grid, modes = (8, 6), (2, 2)
    wl = synth.Workload("tiny", "network", "bf16", 2, grid, modes, 4, in_ch=3, hidden=5,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    monkeypatch.setattr(T, "capi", _FakeLibrary(modes))
    sched = [(0, "bf16"), (2, "f32")]
    a = torch.from_numpy(np.asarray(inp["a"], np.float32))
    t = torch.from_numpy(np.asarray(inp["target"], np.float32))

    def trainer():
        return T.Trainer(grid, modes, 3, 4, inp["params"], T.PrecisionSchedule(sched), hidden=5,
                         n_layers=2, lr=1e-2, weight_decay=0.05, device="cpu")

    straight = trainer()
    for _ in range(4):
        straight.step(a, t)
    first = trainer()
    for _ in range(2):
        first.step(a, t)
    state = first.state_dict()
    resumed = T.Trainer(grid, modes, 3, 4, {**inp["params"]}, T.PrecisionSchedule([(0, "f32")]),
                        hidden=5, n_layers=2, device="cpu")
    resumed.load_state_dict(state)
    assert resumed.step_count == 2 and resumed.schedule.phases == sched
    for _ in range(2):
        resumed.step(a, t)
    assert torch.equal(resumed.master, straight.master)
    assert torch.equal(resumed.m, straight.m) and torch.equal(resumed.v, straight.v)
    with pytest.raises(ValueError):
        T.Trainer(grid, modes, 3, 4, synth.make_network_inputs(
            synth.Workload("w", "network", "f32", 2, grid, modes, 5, in_ch=3, hidden=5,
                           n_layers=2, backward=True))["params"], T.PrecisionSchedule([(0, "f32")]),
            hidden=5, n_layers=2, device="cpu").load_state_dict(state)
