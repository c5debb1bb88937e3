"""fp64 CPU oracle of the TTT-layer forward pass.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline / reference arm, never by the CUDA product path.
"""
from .ttt_oracle import (  # noqa: F401
    chunk_bounds, dwconv_apply, dwconv_weight_grad, forward, forward_head, gelu, gelu_prime,
    inner_backward, inner_forward,
    instance_norm, loss_grad, loss_value, matrix_shapes, newton_schulz, pack, row_l2_normalize,
    silu, silu_prime, unpack, update_chunk,
)
