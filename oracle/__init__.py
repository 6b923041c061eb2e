"""Float64 CPU oracle for ReLU linear attention (test infrastructure).

This package is test infrastructure. Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it. The CUDA library never
calls it, and it shares no code with the CUDA library.

Every function works on float64 numpy arrays. Inputs drawn in bfloat16 are read
as the exact values they hold. See ``oracle/linear_attention.py`` for the
citations of each step.
"""
from .linear_attention import (  # noqa: F401
    HEAD_DIM,
    ROPE_SEGMENTS,
    relu,
    rope_positions,
    rope_angles,
    rope_rotate,
    feature_map,
    state_reduce,
    apply,
    attention,
    attention_bruteforce,
    block_causal_step,
    block_causal_bruteforce,
    apply_rows,
    to_f64,
    rope_unrotate,
    backward,
    causal_attention,
    causal_bruteforce,
)
from .temporal_conv import temporal_conv  # noqa: F401,E402
from .qkv_state import bf16_round, qkv_projection, qkv_state, key_value_heads  # noqa: F401,E402
