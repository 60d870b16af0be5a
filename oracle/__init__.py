"""fp64 CPU oracle of the E2-TTT chunk scan.

TEST INFRASTRUCTURE: imported only by the tests, the smoke check and the
benchmark's CPU baseline. The CUDA library and its binding never use it.
"""
from .e2ttt_oracle import *  # noqa: F401,F403
from .e2ttt_oracle import (LINEAR, SWIGLU, GELU, LOSS_MSE, LOSS_NEG_DOT, seq_fwd, tokenwise_fwd,  # noqa: F401
                           closed_fwd, seq_bwd, closed_bwd, chunk_kernels, all_chunk_kernels,
                           chunk_kernels_vjp, loss_grad, loss_grad_vjp, fast_apply, fast_apply_vjp,
                           loss_value, state_elems, unpack, pack, rel_fro, COEF_PER_TOKEN,
                           COEF_CHUNK_MEAN, chunk_mean_kernels, gelu, dgelu, d2gelu)
