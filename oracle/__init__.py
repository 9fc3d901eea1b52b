"""fp64 CPU oracle for the Gemma-4-style attention layer.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs may import this package.  It is independent of the CUDA library: the two
share no code, header or constant.
"""
from .oracle import (  # noqa: F401
    OracleCfg,
    rope_pairs,
    rmsnorm,
    rope,
    qknorm_rope,
    prefill_rows,
    decode,
    decode_ring,
    prefill_chunk,
    quantize_int8,
    dequantize_int8,
    decode_int8,
    bf16_bits,
)
