"""B200-native paged KV cache: slot-mapped KV write (16-bit, INT8, FP8-e4m3,
asymmetric uint8 with zero points, INT4, FP4-E2M1), block-table decode
attention (GQA, split-KV merged in-kernel, sliding windows), multi-query
attention for speculative verify and chunked prefill (a query-major tcgen05
kernel for long chunks), copy-on-write block copy, and a host block allocator
with automatic prefix caching, behind the C ABI of libpagedkv.so.

The Python layer only marshals arguments; see ``pagedkv`` for the calls.
"""
from .pagedkv import (  # noqa: F401
    KV_FORMATS,
    BlockAllocator,
    NoBlocksError,
    PagedKVError,
    copy_blocks,
    decode_plan,
    device_status,
    kv_cache_write,
    lib,
    multi_query_plan,
    new_workspace,
    paged_attention_decode,
    paged_attention_decode_noalloc,
    paged_attention_multi_query,
    prefix_key,
    set_validation,
    version,
)
