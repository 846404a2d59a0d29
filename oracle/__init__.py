"""CPU fp64 oracle: test infrastructure only (see coda_oracle.py)."""

from .coda_oracle import (  # noqa: F401
    gemm,
    mlp_block_backward,
    mlp_block_forward,
    grg_backward_stored,
    grg_forward_stored,
    round_bf16,
    swiglu_backward_stored,
    swiglu_forward_stored,
    grg_backward,
    grg_forward,
    partial_sumsq,
    qkv_rope_backward,
    qkv_rope_forward,
    rope_angles,
    rope_rotate,
    silu,
    swiglu_backward,
    swiglu_forward,
    xent_backward,
    xent_forward,
)
