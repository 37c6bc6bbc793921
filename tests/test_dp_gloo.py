"""Data-parallel host logic on CPU with world_size 2 (gloo): batch sharding,
the global-mean MSE scaling and the gradient all-reduce reproduce the
single-process full-batch gradients of the network.  The per-rank compute is
the CPU oracle (the logic under test is the sharding and the exchange)."""

import os
import socket

import numpy as np
import pytest

from fourier_neural_spectral_fno_b200 import dp, synth


def test_shard_range_covers_batch():
    for batch in (1, 7, 16, 33):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_range(batch, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == batch
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_range(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    import oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.Workload("dp", "network", "f32", 4, (8, 12), (2, 3), 5, in_ch=3, hidden=7,
                            n_layers=2, backward=True)
        inp = synth.make_network_inputs(wl)
        a, p, tgt = inp["a"], inp["params"], inp["target"]
        lo, hi = dp.shard_range(wl.batch, rank, world)
        u, sv = O.forward(a[lo:hi], p, wl.modes, save=True)
        _, du = O.mse(u, tgt[lo:hi])                 # local mean
        du = du * dp.mse_scale(du.size, tgt.size)    # -> global mean
        g = O.backward(a[lo:hi], p, sv, du, wl.modes)
        grads = {k: ([torch.from_numpy(np.ascontiguousarray(
                        np.stack([x.real, x.imag], -1) if np.iscomplexobj(x) else x)) for x in v]
                     if isinstance(v, list) else torch.from_numpy(np.ascontiguousarray(v)))
                 for k, v in g.items() if k != "a"}
        dp.allreduce_grads(grads)
        if rank == 0:
            flat = dp.flatten(grads).numpy()
            np.save(os.path.join(out_dir, "dp.npy"), flat)
    finally:
        dist.destroy_process_group()


def test_allreduce_matches_full_batch(tmp_path):
    import torch
    import torch.multiprocessing as mp

    import oracle as O
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    flat_dp = np.load(tmp_path / "dp.npy")
    wl = synth.Workload("dp", "network", "f32", 4, (8, 12), (2, 3), 5, in_ch=3, hidden=7,
                        n_layers=2, backward=True)
    inp = synth.make_network_inputs(wl)
    u, sv = O.forward(inp["a"], inp["params"], wl.modes, save=True)
    _, du = O.mse(u, inp["target"])
    g = O.backward(inp["a"], inp["params"], sv, du, wl.modes)
    ref = {k: ([torch.from_numpy(np.ascontiguousarray(
                  np.stack([x.real, x.imag], -1) if np.iscomplexobj(x) else x)) for x in v]
               if isinstance(v, list) else torch.from_numpy(np.ascontiguousarray(v)))
           for k, v in g.items() if k != "a"}
    flat_ref = dp.flatten(ref).numpy()
    np.testing.assert_allclose(flat_dp, flat_ref, rtol=1e-5, atol=1e-7)
