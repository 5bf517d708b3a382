"""fp64 CPU oracle for attention (forward, backward, RoPE) -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product path (the CUDA
library and its Python binding) never does.
"""
from .attn_ref import (  # noqa: F401
    attention_backward,
    attention_backward_rope,
    attention_forward,
    attention_forward_rope,
    attention_rows,
    head_backward,
    head_forward,
    head_scores,
    kv_head,
    rope_angles,
    rope_rotate,
    rope_rotate_transpose,
)
