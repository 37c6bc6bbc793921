"""The bounded waits of the tensor-core pipelines: when a wait runs out, the
kernel records FNO_ERR_TIMEOUT in the library's device error word, drains what
it has in flight and returns, and the GPU stays usable.

The wait limit is lowered to a single probe (fno_set_wait_limit(0)) for one
block forward on the default kernels (the streaming transform and the
pipelined epilogue), whose roles are never all in step at once, so some wait
gives up; nothing is planted on the GPU side.  With the default restored the
next call is correct."""

import numpy as np
import pytest
import torch

import oracle as O
from fourier_neural_spectral_fno_b200 import capi, synth

from fno_testlib import TOL, assert_close, dev, dev_complex, empty, host

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_next_call_is_correct():
    grid, modes, B, C = (256, 256), (16, 16), 2, 32
    rng = np.random.default_rng(31)
    x = synth.quantize(rng.standard_normal((B, C) + grid), "f32")
    r = synth.quantize_complex(synth.spectral_weights(rng, C, C, capi.num_modes(grid, modes)) * C,
                               "f32")
    w = synth.quantize(rng.uniform(-1, 1, (C, C)) / np.sqrt(C), "f32")
    b = synth.quantize(rng.uniform(-0.5, 0.5, C), "f32")
    d = capi.block_desc(B, C, C, grid, modes)
    args = (dev(x), dev_complex(r), dev(w), dev(b))
    prev_path = capi.fno_set_tensor_cores(1)
    capi.fno_device_error(clear=True)
    prev = capi.fno_set_wait_limit(0)
    try:
        assert prev > 0
        y = empty((B, C) + grid)
        capi.fno_block_fwd(d, *args, y)
        torch.cuda.synchronize()
        with pytest.raises(capi.FnoError) as info:
            capi.fno_device_error(clear=True)
        assert info.value.code == capi.FNO_ERR_TIMEOUT
    finally:
        capi.fno_set_wait_limit(prev)
        capi.fno_set_tensor_cores(prev_path)
    assert capi.fno_set_wait_limit(prev) == prev
    capi.fno_device_error(clear=True)        # cleared by the read above: no error now
    y2 = empty((B, C) + grid)
    capi.fno_block_fwd(d, *args, y2)
    capi.fno_device_error(clear=True)
    y_ref, _, _ = O.block_fwd(x, r, w, b, modes)
    assert_close(host(y2), y_ref, TOL["f32"], "y after the expiry")
