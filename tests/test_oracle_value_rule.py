"""Pin of the Value rule: decode over the merged cache equals attention over the
expanded cache.

The KVSlimmer pages merge homogeneous Keys while preserving heterogeneous
Values ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程", 核心判断 and
§数学主线一; AsymKV's lossless value compression on the fugumt related-paper
list). The oracle stores the count-weighted mean value plus log(count) as a
logit bias. Here, after several rounds, each original position is given the
merged key of its group and its OWN original value; textbook attention over
that expanded cache must equal the oracle's decode over the merged cache.
"""

import math

import numpy as np
import pytest

import oracle


def provenance_after_round(groups, selected, c0, length):
    """Map output rows to lists of original positions, by counting."""
    P = len(selected)
    out = [groups[t] for t in range(c0)]
    for p in range(P):
        a, b = c0 + 2 * p, c0 + 2 * p + 1
        if selected[p]:
            out.append(groups[a] + groups[b])
        else:
            out.append(groups[a])
            out.append(groups[b])
    out.extend(groups[t] for t in range(c0 + 2 * P, length))
    return out


def expanded_attention(q, K_rows, V_orig):
    d = len(q)
    e = [float(np.dot(q, K_rows[t])) / math.sqrt(d) for t in range(len(K_rows))]
    m = max(e)
    w = [math.exp(x - m) for x in e]
    z = sum(w)
    return sum(w[t] * V_orig[t] for t in range(len(w))) / z


@pytest.mark.parametrize("seed,ratio", [(0, 2), (1, 4), (2, 8)])
def test_merged_cache_attention_equals_expanded_cache(seed, ratio):
    rng = np.random.default_rng(seed)
    length, d, G, W, c0, n_recent = 120, 6, 2, 4, 8, 4
    K = rng.normal(size=(1, 1, length, d))
    V = rng.normal(size=(1, 1, length, d))
    Q = rng.normal(size=(1, G, W, d)) * 2
    cache = oracle.cache_from_arrays(K, V, np.array([[length]]))
    target = np.array([[length // ratio]])
    out, rounds = oracle.compress(cache, Q, W, np.array([[c0]]), n_recent, target)
    assert len(rounds) >= 2 if ratio > 2 else len(rounds) >= 1
    groups = [[t] for t in range(length)]
    cur_len = length
    for r in rounds:
        groups = provenance_after_round(groups, r.selected[0][0], c0, cur_len)
        cur_len = len(groups)
    assert cur_len == out.length(0, 0)
    counts = np.array([len(g) for g in groups], dtype=np.float64)
    np.testing.assert_allclose(out.log_n[0][0], np.log(counts), rtol=1e-12, atol=1e-12)
    # mean value of each group
    for i, g in enumerate(groups):
        np.testing.assert_allclose(out.V[0][0][i], V[0, 0, g].mean(axis=0), rtol=1e-10, atol=1e-12)
    # expanded cache: original position t gets its group's merged key and its own value
    key_of = np.zeros((length, d))
    for i, g in enumerate(groups):
        for t in g:
            key_of[t] = out.K[0][0][i]
    q = rng.normal(size=(G, d)) * 2
    merged = oracle.decode_attention(q, out.K[0][0], out.V[0][0], out.log_n[0][0], out.length(0, 0))
    for g in range(G):
        np.testing.assert_allclose(merged[g], expanded_attention(q[g], key_of, V[0, 0]),
                                   rtol=1e-10, atol=1e-12)
