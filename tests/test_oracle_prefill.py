"""Pins of the oracle's chunked streaming prefill compression.

The KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
§实验设置) runs with a compression context budget of 2048 tokens, chunks of 512 and
32 preserved initial tokens; the loop is: append a chunk, merge back to the budget.
Here the loop is checked against facts that do not depend on which pairs it picks:
lengths, the total count of prompt tokens the cache stands for, the untouched
protected rows, no change when the budget is never exceeded, and the Value rule
(attention over the merged cache equals attention over the expanded cache, every
original position keeping its own value under its group's merged key).
"""

import numpy as np
import pytest

import oracle
from test_oracle_value_rule import expanded_attention, provenance_after_round


def _prompt(seed, T, d=8, H=2, G=2, W=4):
    rng = np.random.default_rng(seed)
    K = rng.normal(size=(1, H, T, d))
    V = rng.normal(size=(1, H, T, d))
    Q = rng.normal(size=(1, H * G, T, d)) * 2        # a query per position
    return K, V, Q


def _run(K, V, Q, chunk, budget, sink, W, form="full"):
    B, H, T, d = K.shape
    cache = oracle.cache_from_arrays(np.zeros((B, H, 0, d)), np.zeros((B, H, 0, d)),
                                     np.zeros((B, H), dtype=np.int64))
    history = []
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        Qw = Q[:, :, c1 - W:c1]
        cache, rounds = oracle.prefill_chunk(cache, K[:, :, c0:c1], V[:, :, c0:c1], Qw, W, budget,
                                             sink, form=form)
        history.append((c1, cache, rounds))
    return cache, history


@pytest.mark.parametrize("chunk,budget", [(16, 40), (24, 40), (10, 64)])
def test_lengths_counts_and_protected_rows(chunk, budget):
    sink, W = 4, 4
    K, V, Q = _prompt(1, 150, W=W)
    _, history = _run(K, V, Q, chunk, budget, sink, W)
    for c1, cache, _ in history:
        for h in range(cache.H):
            L = cache.length(0, h)
            assert L == min(c1, budget)
            # every prompt token so far is stood for exactly once
            assert np.sum(np.exp(cache.log_n[0][h])) == pytest.approx(c1, rel=1e-12)
            # the preserved initial rows and the newest W rows are the prompt's own
            np.testing.assert_array_equal(cache.K[0][h][:sink], K[0, h, :sink])
            np.testing.assert_array_equal(cache.K[0][h][L - W:], K[0, h, c1 - W:c1])
            np.testing.assert_array_equal(cache.V[0][h][L - W:], V[0, h, c1 - W:c1])
            np.testing.assert_array_equal(cache.log_n[0][h][L - W:], 0.0)


def test_no_merge_while_the_budget_holds():
    K, V, Q = _prompt(2, 90)
    cache, history = _run(K, V, Q, chunk=32, budget=128, sink=4, W=4)
    assert all(len(r) == 0 for _, _, r in history)
    for h in range(2):
        np.testing.assert_array_equal(cache.K[0][h], K[0, h])
        np.testing.assert_array_equal(cache.V[0][h], V[0, h])
        np.testing.assert_array_equal(cache.log_n[0][h], 0.0)


@pytest.mark.parametrize("seed", [3, 4])
def test_value_rule_holds_through_the_chunked_loop(seed):
    sink, W, chunk, budget = 4, 4, 20, 36
    K, V, Q = _prompt(seed, 130, W=W)
    cache, history = _run(K, V, Q, chunk, budget, sink, W)
    h = 1
    groups, prev = [], 0
    for c1, _, rounds in history:
        groups = groups + [[t] for t in range(prev, c1)]
        for r in rounds:
            groups = provenance_after_round(groups, r.selected[0][h], sink, len(groups))
        prev = c1
    assert len(groups) == cache.length(0, h)
    assert sorted(t for g in groups for t in g) == list(range(130))
    for g in groups:                                   # groups are runs of adjacent positions
        assert g == list(range(g[0], g[0] + len(g)))
    key_of = np.zeros((130, K.shape[3]))
    for i, g in enumerate(groups):
        for t in g:
            key_of[t] = cache.K[0][h][i]
    q = np.random.default_rng(seed).normal(size=(2, K.shape[3])) * 2
    merged = oracle.decode_attention(q, cache.K[0][h], cache.V[0][h], cache.log_n[0][h],
                                     cache.length(0, h))
    for g in range(2):
        np.testing.assert_allclose(merged[g], expanded_attention(q[g], key_of, V[0, h]),
                                   rtol=1e-10, atol=1e-12)


def test_chunked_loop_invariants_for_random_settings():
    """Property check over random prompt lengths, chunk sizes and budgets: after every
    chunk each head holds min(tokens so far, budget) rows standing for exactly the tokens
    so far, with the preserved initial rows and the newest W rows untouched."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=20, deadline=None)
    @given(T=st.integers(40, 160), chunk=st.integers(4, 48), sink=st.integers(0, 8),
           W=st.integers(1, 6), extra=st.integers(1, 60), seed=st.integers(0, 10_000))
    def check(T, chunk, sink, W, extra, seed):
        budget = sink + W + extra
        if chunk < W:
            return                                    # the window lies inside the chunk
        K, V, Q = _prompt(seed, T, d=4, H=1, G=1, W=W)
        _, history = _run(K, V, Q, chunk, budget, sink, W)
        for c1, cache, _ in history:
            L = cache.length(0, 0)
            assert L == min(c1, budget)
            assert np.sum(np.exp(cache.log_n[0][0])) == pytest.approx(c1, rel=1e-12)
            keep = min(sink, L)
            np.testing.assert_array_equal(cache.K[0][0][:keep], K[0, 0, :keep])
            np.testing.assert_array_equal(cache.K[0][0][L - W:], K[0, 0, c1 - W:c1])

    check()
