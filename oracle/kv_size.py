"""KV-cache size arithmetic (oracle; test infrastructure only).

"LLM 推理优化深度解析" (blog.longjiangtao.top), §KV Cache 的本质, states the
cache size as the product of a factor 2 (one K and one V), the layer count,
the KV-head count, the head dimension, the sequence length, the bytes per
element and the batch size, and works it for Llama-2-7B (32 layers, 32 heads,
head_dim 128, fp16) at 4096 tokens.  "KV Cache 与 PagedAttention"
(ai-infra-wiki), §KV cache 有多大, gives the per-layer, per-token form
2 x n_kv x head_dim x 2 bytes for 16-bit values.
"""


def kv_cache_bytes(n_layers, n_kv_heads, head_dim, seq_len, batch=1, bytes_per_elt=2):
    """Bytes of K plus V for ``batch`` sequences of ``seq_len`` tokens."""
    return 2 * n_layers * n_kv_heads * head_dim * seq_len * bytes_per_elt * batch


def kv_bytes_per_token_per_layer(n_kv_heads, head_dim, bytes_per_elt=2):
    """Bytes one token adds to one layer's cache (K and V)."""
    return 2 * n_kv_heads * head_dim * bytes_per_elt


def decode_tokens_per_s_bound(bandwidth_gb_s, bytes_read_per_token_gb):
    """Upper bound on single-stream decode rate when each token must read
    ``bytes_read_per_token_gb`` from memory at ``bandwidth_gb_s``
    ("LLM 推理优化深度解析", §Decode（解码）阶段)."""
    return bandwidth_gb_s / bytes_read_per_token_gb


def paged_blocks_needed(seq_len, block_size=16):
    """Physical blocks a sequence of ``seq_len`` tokens occupies when blocks
    are allocated on demand: ceil(seq_len / block_size)."""
    return (seq_len + block_size - 1) // block_size


def paged_waste_tokens(seq_len, block_size=16):
    """Unused token slots in a sequence's last block (internal fragmentation);
    the pages bound it by one block ("LLM 推理优化深度解析", §PagedAttention
    table: 最多浪费一个块)."""
    return paged_blocks_needed(seq_len, block_size) * block_size - seq_len
