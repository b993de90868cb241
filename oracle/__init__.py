"""fp64 CPU oracle for the exact RoPE-attention loss and its closed-form gradient.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import or run it.  It shares no code with the CUDA path.

Every function is a plain, slow, literal restatement of a definition, in float64
NumPy, row-blocked over queries so that no n x n array is ever held.  See
``oracle.rope_attention`` for the definitions and the passages they follow.
"""
from .rope_attention import (  # noqa: F401
    rope_theta,
    rope_angles,
    rope_rotate,
    softmax_rows,
    gamma_closed_form,
    instance_forward_backward,
    instance_loss,
    forward_backward,
    loss_only,
    scores_rows,
    forward_rows,
    rotation_matrix,
    combined_weight_literal,
    combined_weight_forward_backward,
    poly_exp,
    poly_features,
    approx_instance_forward_backward,
    approx_forward_backward,
    ORACLE_PARITY_PINNED,
)
