"""CPU oracle for paged KV attention -- test infrastructure only.

Imported by tests, the smoke check and the benchmark's CPU-baseline leg; never
by the library.  See ``oracle.paged_attention`` for what it computes and which
passages it follows.
"""
from .paged_attention import (  # noqa: F401
    bf16_bits_to_f64,
    chunked_prefill_attention,
    decode_attention,
    decode_partials,
    gather_request_kv,
    kv_append,
    split_k_combine,
)
