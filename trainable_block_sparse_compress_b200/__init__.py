"""InfLLM v2 block-sparse attention for B200 (sm_100a).

The computation runs in ``libinfllmv2.so`` (hand-written CUDA, C ABI in
``include/infllmv2.h``); this package is its thin Python binding plus the seeded
synthetic-input generator used by the tests and the benchmark.
"""
from .ops import (  # noqa: F401
    Params,
    append_kv,
    compress_keys,
    decode,
    device_error,
    num_blocks,
    num_kernels,
    prefill,
    prefill_chunk,
    select_blocks_chunk,
    sparse_attn_backward,
    sparse_attn_chunk,
    select_blocks_decode,
    select_blocks_prefill,
    sparse_attn_decode,
    sparse_attn_decode_noalloc,
    sparse_attn_prefill,
    workspace_size,
)
