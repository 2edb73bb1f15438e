"""Pins of the oracle's selection, budget and compaction against brute force.

The pages leave pair selection and the budget rule open; the oracle's reading
(R smallest (score, index), rounds until the budget is met exactly) is pinned
here by exhaustive search and by counting on tiny inputs.
"""

import itertools
import math

import numpy as np
import pytest

import oracle


def brute_force_select(scores, R):
    """Among all R-subsets minimise (sum of scores, sorted index tuple)."""
    best = None
    for sub in itertools.combinations(range(len(scores)), R):
        key = (sum(scores[i] for i in sub), sub)
        if best is None or key < best:
            best = key
    mask = np.zeros(len(scores), dtype=bool)
    mask[list(best[1])] = True
    return mask


@pytest.mark.parametrize("seed", range(8))
def test_selection_equals_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    P = int(rng.integers(1, 11))
    scores = rng.integers(-3, 4, size=P).astype(np.float64)   # integer values: ties, exact sums
    for R in range(P + 1):
        assert np.array_equal(oracle.select_pairs(scores, R), brute_force_select(list(scores), R))


def test_nan_scores_rank_last_like_infinity():
    scores = np.array([np.nan, 1.0, np.inf, -1.0, np.nan, 0.0])
    assert list(np.flatnonzero(oracle.select_pairs(scores, 3))) == [1, 3, 5]
    # among the +inf / NaN keys, lower index first
    assert list(np.flatnonzero(oracle.select_pairs(scores, 4))) == [0, 1, 3, 5]
    assert list(np.flatnonzero(oracle.select_pairs(scores, 5))) == [0, 1, 2, 3, 5]


def test_selection_rejects_infeasible_counts():
    with pytest.raises(ValueError):
        oracle.select_pairs(np.zeros(3), 4)
    with pytest.raises(ValueError):
        oracle.select_pairs(np.zeros(3), -1)


def _position_cache(length, d=3):
    """Rows encode their position so order and provenance can be read back."""
    K = np.array([[t, 2 * t, 0.5] for t in range(length)], dtype=np.float64)[:, :d]
    V = -K
    return K, V


@pytest.mark.parametrize("length,c0,n_recent", [(20, 4, 3), (21, 0, 0), (9, 2, 2), (7, 7, 0),
                                                (5, 0, 5), (33, 32, 0)])
def test_offsets_and_length_by_counting(length, c0, n_recent):
    rng = np.random.default_rng(length + c0)
    K, V = _position_cache(length)
    P = oracle.num_pairs(length, c0, n_recent)
    assert P == max(0, (length - n_recent - c0) // 2)
    sel = rng.random(P) < 0.5
    w = rng.random(P)
    m = oracle.merge_compact_head(K, V, None, length, c0, n_recent, sel, w)
    assert m.length == length - int(sel.sum())
    for p in range(P):
        expect = c0 + sum(1 if sel[i] else 2 for i in range(p))
        assert m.out_offset[p] == expect
    # prefix and suffix copied, order preserved
    assert np.array_equal(m.K[:c0], K[:c0])
    tail = length - (c0 + 2 * P)
    if tail:
        assert np.array_equal(m.K[-tail:], K[-tail:])
    firsts = m.K[:, 0]
    assert np.all(np.diff(firsts) > 0)


def test_zero_merges_leave_the_cache_unchanged():
    rng = np.random.default_rng(1)
    K, V = rng.normal(size=(2, 40, 8))
    ln = rng.random(40)
    m = oracle.merge_compact_head(K, V, ln, 40, 32, 0, np.zeros(4, bool), rng.random(4))
    assert np.array_equal(m.K, K) and np.array_equal(m.V, V) and np.array_equal(m.log_n, ln)


def test_value_merge_uses_counts_and_log_count():
    K = np.zeros((4, 2))
    V = np.array([[1.0, 0.0], [0.0, 4.0], [2.0, 2.0], [0.0, 0.0]])
    ln = np.array([math.log(3.0), 0.0, 0.0, math.log(5.0)])
    m = oracle.merge_compact_head(K, V, ln, 4, 0, 0, np.array([True, True]), np.array([0.5, 0.5]))
    np.testing.assert_allclose(m.V[0], [3 / 4, 1.0])
    np.testing.assert_allclose(m.V[1], [2 / 6, 2 / 6])
    np.testing.assert_allclose(m.log_n, [math.log(4.0), math.log(6.0)])


@pytest.mark.parametrize("length,c0,n_recent,ratio", [(512, 32, 32, 2), (300, 32, 32, 4),
                                                      (1001, 32, 32, 8), (130, 3, 5, 2)])
def test_round_driver_reaches_the_budget_exactly(length, c0, n_recent, ratio):
    rng = np.random.default_rng(length)
    d, G, W = 4, 2, 4
    K = rng.normal(size=(1, 2, length, d))
    V = rng.normal(size=(1, 2, length, d))
    Q = rng.normal(size=(1, 2 * G, W, d))
    cache = oracle.cache_from_arrays(K, V, np.full((1, 2), length))
    target = np.full((1, 2), oracle.budget(length, ratio))
    out, rounds = oracle.compress(cache, Q, W, np.full((1, 2), c0), n_recent, target)
    assert np.all(out.lengths() == target)
    # every round but the last merges every candidate pair
    for r in rounds[:-1]:
        P = [[s.score.shape[0] for s in row] for row in r.scores]
        assert np.array_equal(r.R, np.array(P))


def test_pooled_scope_budget_and_global_selection():
    rng = np.random.default_rng(9)
    d, H, G, W, length = 4, 3, 2, 4, 96
    K = rng.normal(size=(2, H, length, d))
    V = rng.normal(size=(2, H, length, d))
    Q = rng.normal(size=(2, H * G, W, d))
    cache = oracle.cache_from_arrays(K, V, np.full((2, H), length))
    target = np.array([H * length // 2, H * length // 2 - 5])
    out, rounds = oracle.compress(cache, Q, W, np.full((2, H), 8), 4, target, scope="pooled")
    assert np.array_equal(out.lengths().sum(axis=1), target)
    last = rounds[-1]
    for b in range(2):
        pooled = np.concatenate([last.scores[b][h].score for h in range(H)])
        chosen = np.concatenate([last.selected[b][h] for h in range(H)])
        R = int(chosen.sum())
        assert R == last.R[b]
        # exactly the R smallest of the pooled scores
        assert np.all(pooled[chosen].max(initial=-np.inf) <= pooled[~chosen].min(initial=np.inf))


def test_storage_rounding_matches_torch_conversions():
    import torch
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(size=2000) * 10.0 ** rng.integers(-8, 8, size=2000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.001953125, 65504.0, 3.0e38]])
    for storage, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        ref = torch.tensor(x, dtype=torch.float64).to(torch.float32).to(tdt).to(torch.float64).numpy()
        got = oracle.storage_round(x, storage)
        assert np.array_equal(got, ref), storage
