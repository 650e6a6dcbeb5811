"""CPU oracle for the Grok-1 MoE feed-forward sublayer.

TEST INFRASTRUCTURE ONLY. This package is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``, and by nothing else. The product path (the CUDA library
and its Python binding) never imports, links or executes anything here; it
fails loudly when the CUDA extension is missing instead of falling back.
"""

from .moe_oracle import (  # noqa: F401
    ACTIVATIONS,
    GELU_MODES,
    dequant_int8,
    dispatch,
    expert_ffn,
    ffn_size,
    forward_dense_bruteforce,
    forward_sparse,
    gelu_erf,
    gelu_tanh,
    near_tie_mask,
    post_norm_residual,
    route,
    route_alternatives,
    silu,
    softmax_fp64,
)
