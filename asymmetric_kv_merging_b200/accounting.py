"""Byte accounting for caches and for the roofline of each kernel.

Plain arithmetic on shapes; no device work. The per-token cache size follows
the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
§算一遍：KV cache 为什么值得压): layers x 2 (K and V) x KV heads x head dim x
bytes per element.
"""


def kv_cache_bytes(layers, kv_heads, head_dim, elem_bytes, tokens, batch=1):
    """Bytes of a K+V cache holding `tokens` tokens for each of `batch` sequences."""
    return int(layers) * 2 * int(kv_heads) * int(head_dim) * int(elem_bytes) * int(tokens) * int(batch)


def decode_bytes_per_token(head_dim, elem_bytes):
    """Algorithmic bytes one decode step reads per cached token per KV head:
    its key and value rows plus its fp32 log-count."""
    return 2 * int(head_dim) * int(elem_bytes) + 4


def merge_bytes(n_in, n_out, head_dim, elem_bytes):
    """Algorithmic bytes of one merge-compaction pass over one KV head: read
    every input row of K and V and its log-count, write every output row."""
    row = 2 * int(head_dim) * int(elem_bytes) + 4
    return int(n_in) * row + int(n_out) * row
