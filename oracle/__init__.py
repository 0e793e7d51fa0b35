"""FP64 CPU oracle (test infrastructure only; see ``oracle.attention``).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package. The CUDA library never calls it.
"""
from .attention import (  # noqa: F401
    HEAD_DIM,
    allowed_chunk,
    allowed_from_bits,
    allowed_full,
    allowed_range,
    attention,
    attention_head,
    cross_attention,
    dequantize_q8_0,
    encoder_attention,
    packed_bias,
    qkv_projection,
    qkv_projection_q8_0,
    range_attention,
    slotmask_attention,
)
