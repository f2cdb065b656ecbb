"""B200-native paged KV cache decode: slot-mapped KV write, block-table decode
attention (GQA, split-KV), copy-on-write block copy, INT8 / FP8-e4m3 KV
storage, and a host block allocator, behind the C ABI of libpagedkv.so.

The Python layer only marshals arguments; see ``pagedkv`` for the calls.
"""
from .pagedkv import (  # noqa: F401
    BlockAllocator,
    NoBlocksError,
    PagedKVError,
    copy_blocks,
    decode_plan,
    device_status,
    kv_cache_write,
    lib,
    paged_attention_decode,
    set_validation,
    version,
)
