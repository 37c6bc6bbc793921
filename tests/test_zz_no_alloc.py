"""The allocation-free spectral forward (fno_spectral_conv_fwd_noalloc).

Callers such as plugins that own no allocator, or code where a cudaMalloc
would stall or is not allowed, can run the spectral convolution with only
their inputs and outputs: the scratch is a fixed array inside the library.
This file is collected last on purpose, and it must pass both alone in a fresh
process and after every other test.  It checks the result against the
workspace-taking entry point, on two calls in a row (the second call finds the
array holding the first call's leftovers), and that an oversized problem is
refused."""

import numpy as np
import pytest
import torch

from fourier_neural_spectral_fno_b200 import capi, synth

from fno_testlib import TOL, assert_close, dev, dev_complex, empty, host, host_complex

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("grid,modes,dtype", [((256, 256), (16, 16), "f32"),
                                              ((70, 130), (6, 9), "f32"),
                                              ((64, 64), (10, 12), "bf16")])
def test_noalloc_matches_workspace_entry_point_twice(grid, modes, dtype):
    rng = np.random.default_rng(21)
    b, ci, co = 4, 8, 6
    k = capi.num_modes(grid, modes)
    d = capi.block_desc(b, ci, co, grid, modes, dtype)
    assert capi.fno_workspace_size(d, capi.FNO_OP_SPECTRAL_FWD) <= capi.FNO_NOALLOC_SCRATCH_BYTES
    for call in range(2):
        x = dev(synth.quantize(rng.standard_normal((b, ci) + grid), dtype), dtype)
        r = dev_complex(synth.quantize_complex(
            rng.standard_normal((ci, co, k)) + 1j * rng.standard_normal((ci, co, k)), dtype), dtype)
        y_ref, xh_ref = empty((b, co) + grid, dtype), empty((b, ci, k, 2))
        capi.fno_spectral_conv_fwd(d, x, r, y_ref, xh_ref)
        y, xh = empty((b, co) + grid, dtype), empty((b, ci, k, 2))
        capi.fno_spectral_conv_fwd_noalloc(d, x, r, y, xh)
        assert_close(host(y), host(y_ref), TOL[dtype], f"y (call {call})")
        assert_close(host_complex(xh), host_complex(xh_ref), TOL[dtype], f"xhat (call {call})")
        # the same kernels run on the same inputs, so the results are identical
        assert torch.equal(y, y_ref), f"y differs bitwise (call {call})"
        assert torch.equal(xh, xh_ref), f"xhat differs bitwise (call {call})"


def test_noalloc_rejects_problems_beyond_the_scratch():
    d = capi.block_desc(64, 64, 64, (512, 512), (32, 32), "f32")
    need = capi.fno_workspace_size(d, capi.FNO_OP_SPECTRAL_FWD)
    assert need > capi.FNO_NOALLOC_SCRATCH_BYTES
    x = empty((1,))
    with pytest.raises(capi.FnoError) as info:
        capi.fno_spectral_conv_fwd_noalloc(d, x, x, x)
    assert info.value.code == capi.FNO_ERR_WORKSPACE
    assert "built-in scratch" in str(info.value)
