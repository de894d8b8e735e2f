"""CPU oracle for streaming KV-cache attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package. The product library never does.
"""
from .stream_oracle import (  # noqa: F401
    StreamOracle,
    ViewMajorWindow,
    bf16_bits_to_f64,
    bf16_round,
    frame_attention,
    project_kv,
    masked_attention,
    rope_frequencies,
    rope_rotate,
    visible_mask,
)
