"""CPU float64 oracle (test infrastructure only; see ``fno_oracle``)."""
from .fno_oracle import *  # noqa: F401,F403
from .fno_oracle import (axis_wavenumbers, kept_shape, num_modes, mode_weights,
                         truncated_dft, inverse_sum, gelu, gelu_grad,
                         spectral_conv_fwd, spectral_conv_bwd, block_fwd,
                         block_bwd, forward, backward, mse, lift, projection,
                         round_to_storage, adam_update, dtype_at, train,
                         cp_weights, spectral_conv_fwd_cp, cp_factor_grads,
                         spectral_conv_bwd_cp,
                         TANH_PREACT, NO_ACT)
