"""CPU oracle (numpy, float64 by default) for the TTT inner loop.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check in
__graft_entry__ and by the benchmark's cpu_baseline / reference leg.  The
product path never imports it, and it imports nothing from the product.
"""
from .ttt_oracle import *  # noqa: F401,F403
from . import swa_oracle  # noqa: F401
from .ttt_oracle import (Model, make_model, prefill, prefill_sequence, scalar_kernels,  # noqa: F401
                         scalar_kernels_ratio_form, chunk_update_closed, chunk_update_explicit,
                         chunk_update_lact, scalar_heads, recon_forward, recon_chunk, prefill_recon,
                         layer_norm, layer_norm_backward, recon_shapes,
                         token_losses, token_gradients, unpack_blocks, pack_blocks,
                         final_prediction, group_means, state_without_gradients)
