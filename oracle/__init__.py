"""fp64 CPU oracle for exact attention (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` use this package. It shares no code with the CUDA library.
"""

from .attention import (  # noqa: F401
    alibi_bias,
    attention_bwd,
    attention_fwd,
    attention_fwd_fp8,
    decode_e4m3,
    head_probs,
    head_bwd,
    head_fwd,
    dequantize_int8,
    kvcache_decode,
    kvcache_decode_int4,
    kvcache_decode_int8,
    lse_combine,
    pack_int4,
    quantize_int4,
    quantize_int8,
    unpack_int4,
    rotary,
    round_to,
    scores,
    visible_mask,
)
