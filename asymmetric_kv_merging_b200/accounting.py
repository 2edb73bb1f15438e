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


def score_bytes(n_rows, n_pairs, head_dim, elem_bytes, fused=True):
    """Algorithmic bytes of one scoring call over one KV head of n_rows rows with n_pairs
    candidate pairs (2 n_pairs candidate rows).

    fused (the tensor-core passes of bf16 caches): window pass A reads every row's K, V and
    log-count (the window outputs need V); pass B reads the candidate rows' K, V and
    log-counts (the window mass needs K, the pair terms V) and writes a score and a weight
    per pair. Not fused (the CUDA-core path of fp32 caches): the window pass reads every
    row's K, V and log-count, the window-mass pass every row's K and log-count and writes
    the mass, and pair scoring reads the candidate rows' K, V and mass and writes the
    score and weight."""
    k_row = int(head_dim) * int(elem_bytes)
    rows, cand = int(n_rows), 2 * int(n_pairs)
    out = int(n_pairs) * 8
    if fused:
        return rows * (2 * k_row + 4) + cand * (2 * k_row + 4) + out
    return rows * (2 * k_row + 4) + rows * (k_row + 4 + 4) + cand * (2 * k_row + 4) + out


def prefill_chunk_bytes(L, n, budget, sink, W, head_dim, elem_bytes, fused=True):
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
        total += score_bytes(length, P, head_dim, elem_bytes, fused)
        total += merge_bytes(length - sink, length - R - sink, head_dim, elem_bytes)
        length -= R
        rounds += 1
    return total, rounds
