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


def score_bytes(n_rows, n_pairs, head_dim, elem_bytes):
    """Algorithmic bytes of one scoring pass over one KV head of n_rows rows: window
    pass A reads K and the log-counts, pass B reads K, V and the log-counts and writes
    the window mass, pair scoring reads K, V and the window mass and writes a score and
    a weight per pair."""
    k_row = int(head_dim) * int(elem_bytes)
    pass_a = int(n_rows) * (k_row + 4)
    pass_b = int(n_rows) * (2 * k_row + 4 + 4)
    pairs = int(n_rows) * (2 * k_row + 4) + int(n_pairs) * 8
    return pass_a + pass_b + pairs


def prefill_chunk_bytes(L, n, budget, sink, W, head_dim, elem_bytes):
    """Algorithmic bytes of one chunked-prefill step over one KV head that holds L rows:
    append n rows (read the chunk's K and V, write them and their log-counts), then
    the merge rounds back to `budget` (each a scoring pass and an in-place merge over
    the rows from `sink` on). Returns (bytes, rounds)."""
    row = 2 * int(head_dim) * int(elem_bytes)
    total = int(n) * (2 * row + 4)
    length, rounds = int(L) + int(n), 0
    while length > budget:
        P = max(0, (length - W - sink) // 2)
        R = min(P, length - budget)
        if R <= 0:
            raise ValueError("budget unreachable")
        total += score_bytes(length, P, head_dim, elem_bytes)
        total += merge_bytes(length - sink, length - R - sink, head_dim, elem_bytes)
        length -= R
        rounds += 1
    return total, rounds
